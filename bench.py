"""Throughput of the chunked fast-weight update-and-read on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the operation over one batch of synthetic input (default workload: the
associative linear-attention mode, B=4 H=16 T=65536 d=128 C=64, bf16: of the single-GPU
workloads it moves the most tokens and bytes per call). Inputs are
resident in HBM when timing starts; L2 is flushed (a 512 MiB write) before every timed step.
Each step is bracketed by CUDA events on the launching stream; the sum over K steps, max over
ranks, is the timed region, itself bracketed by a barrier and a device synchronize.

Multi-GPU (torchrun, one process per GPU): every (batch, head) stream is independent, so each rank
runs its own batch with no data-path collective (weak scaling); NCCL is used only for the barrier
and the max-over-ranks reduction of the timings.

--impl reference times the fp64 CPU oracle (the deliberately slow reference arm) on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TTT-layer fwd tokens/s on 1 B200; % of bf16 tensor-peak/HBM roofline"
# the backward of the associative mode is measured the same way, as backward tokens/s
METRIC_BWD = "TTT-layer bwd tokens/s on 1 B200; % of bf16 tensor-peak/HBM roofline"


def metric_of(w) -> str:
    return METRIC_BWD if w.kind.endswith("_bwd") else METRIC
DEFAULT_WORKLOAD = "assoc_bf16_B4H16T65536_d128C64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DOMINANT_KERNEL = {"dual": ("dual_tc_kernel", "dual_tc.cu"),
                   "dual_seg": ("dual_tc_kernel", "dual_tc.cu"),
                   "assoc": ("assoc_chunk_kernel", "assoc_scan.cu"),
                   "inplace": ("inplace_chunk_kernel", "inplace_ttt.cu"),
                   "assoc_bwd": ("assoc_yz_kernel", "assoc_yz.cu"),
                   "dual_bwd": ("dual_bwd_tc_kernel", "dual_bwd_tc.cu"),
                   "dual_seg_bwd": ("dual_bwd_tc_kernel", "dual_bwd_tc.cu"),
                   "assoc_momentum": ("mom_chunk_kernel", "assoc_mom.cu"),
                   "inplace_lm": ("inplace_chunk_kernel", "inplace_ttt.cu")}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(fname: str) -> str:
    path = os.path.join(ROOT, "weight_linear_attention_ttt_b200", "csrc", fname)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(workload: str, kernel: str, sha: str):
    """(DRAM bytes, scope) from a committed ncu summary, valid only for the same kernel source
    (profiles/dram_traffic.txt: `workload kernel source_sha256_16 bytes [launch|call]`), else
    (None, None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None, None
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == workload and f[1] == kernel \
                and f[2] == sha:
            return float(f[3]), (f[4] if len(f) > 4 else "launch")
    return None, None


# ----------------------------------------------------------------------------- clocks (NVML)
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: clocks are reported as unavailable
            self.error = str(e)

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = get_reasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workload calls
def make_call(w, x, stream_outputs=None):
    """Returns step() -> outputs, running the whole operation once on the current stream."""
    import torch

    import weight_linear_attention_ttt_b200 as ttt
    from weight_linear_attention_ttt_b200 import inputs as inp

    if w.kind == "dual":
        O = torch.empty_like(x["Q"])
        W = torch.empty((w.B, w.H, w.d, w.d), device=x["Q"].device, dtype=torch.float32)
        return lambda: ttt.ttt_linear_dual_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"], C=w.C,
                                               eta_scalar=x["eta_scalar"], O=O, W_out=W)
    if w.kind == "dual_seg":
        O = torch.empty_like(x["Q"])
        W = torch.empty((w.B, w.H, w.d, w.d), device=x["Q"].device, dtype=torch.float32)
        lib = ttt.load_library()
        nbytes = lib.ttt_linear_dual_seg_workspace_size(w.B, w.H, w.T, w.d, w.C, 1, 0)
        ws = torch.empty(max(nbytes, 16), device=x["Q"].device, dtype=torch.uint8)
        return lambda: ttt.ttt_linear_dual_seg_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"],
                                                   C=w.C, segments=0,
                                                   eta_scalar=x["eta_scalar"], O=O, W_out=W,
                                                   workspace=ws)
    if w.kind == "assoc":
        O = torch.empty_like(x["Q"])
        S = torch.empty((w.B, w.H, w.d, w.d), device=x["Q"].device, dtype=torch.float32)
        lib = ttt.load_library()
        nbytes = lib.ttt_assoc_scan_workspace_size(w.B, w.H, w.T, w.d, w.C, 1)
        ws = torch.empty(max(nbytes, 16), device=x["Q"].device, dtype=torch.uint8)
        return lambda: ttt.ttt_assoc_scan_fwd(x["Q"], x["K"], x["V"], x["eta"], None, C=w.C,
                                              eta_scalar=x["eta_scalar"], O=O, S_out=S,
                                              workspace=ws)
    if w.kind == "assoc_momentum":
        dev = x["Q"].device
        O = torch.empty_like(x["Q"])
        S = torch.empty((w.B, w.H, w.d, w.d), device=dev, dtype=torch.float32)
        M = torch.empty_like(S)
        lib = ttt.load_library()
        nbytes = lib.ttt_assoc_momentum_workspace_size(w.B, w.H, w.T, w.d, w.C, 1)
        ws = torch.empty(max(nbytes, 16), device=dev, dtype=torch.uint8)
        return lambda: ttt.ttt_assoc_momentum_fwd(x["Q"], x["K"], x["V"], x["eta"],
                                                  inp.MOMENTUM_BETA, None, None, C=w.C,
                                                  eta_scalar=x["eta_scalar"], O=O, S_out=S,
                                                  M_out=M, workspace=ws)
    if w.kind == "assoc_bwd":
        dev = x["Q"].device
        outs = dict(dQ=torch.empty_like(x["Q"]), dK=torch.empty_like(x["Q"]),
                    dV=torch.empty_like(x["Q"]),
                    deta=torch.empty((w.B, w.H, w.T), device=dev, dtype=torch.float32),
                    dS0=torch.empty((w.B, w.H, w.d, w.d), device=dev, dtype=torch.float32))
        lib = ttt.load_library()
        nbytes = lib.ttt_assoc_scan_bwd_workspace_size(w.B, w.H, w.T, w.d, w.C, 1)
        ws = torch.empty(max(nbytes, 16), device=dev, dtype=torch.uint8)
        return lambda: ttt.ttt_assoc_scan_bwd(x["Q"], x["K"], x["V"], x["eta"], None, x["dO"],
                                              x["dS_out"], C=w.C, eta_scalar=x["eta_scalar"],
                                              workspace=ws, **outs)
    if w.kind == "dual_seg_bwd":
        dev = x["Q"].device
        outs = dict(dQ=torch.empty_like(x["Q"]), dK=torch.empty_like(x["Q"]),
                    dV=torch.empty_like(x["Q"]),
                    deta=torch.empty((w.B, w.H, w.T), device=dev, dtype=torch.float32),
                    dW0=torch.empty((w.B, w.H, w.d, w.d), device=dev, dtype=torch.float32))
        lib = ttt.load_library()
        nbytes = lib.ttt_linear_dual_seg_bwd_workspace_size(w.B, w.H, w.T, w.d, w.C, 1, 0)
        ws = torch.empty(max(nbytes, 16), device=dev, dtype=torch.uint8)
        return lambda: ttt.ttt_linear_dual_seg_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"],
                                                   x["dO"], x["dW_out"], C=w.C, segments=0,
                                                   eta_scalar=x["eta_scalar"], workspace=ws,
                                                   **outs)
    if w.kind == "dual_bwd":
        dev = x["Q"].device
        outs = dict(dQ=torch.empty_like(x["Q"]), dK=torch.empty_like(x["Q"]),
                    dV=torch.empty_like(x["Q"]),
                    deta=torch.empty((w.B, w.H, w.T), device=dev, dtype=torch.float32),
                    dW0=torch.empty((w.B, w.H, w.d, w.d), device=dev, dtype=torch.float32))
        lib = ttt.load_library()
        nbytes = lib.ttt_linear_dual_bwd_workspace_size(w.B, w.H, w.T, w.d, w.C, 1)
        ws = torch.empty(max(nbytes, 16), device=dev, dtype=torch.uint8)
        return lambda: ttt.ttt_linear_dual_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W0"],
                                               x["dO"], x["dW_out"], C=w.C,
                                               eta_scalar=x["eta_scalar"], workspace=ws, **outs)
    if w.kind == "inplace_lm":
        O = torch.empty((w.T, w.D), device=x["Z"].device, dtype=torch.bfloat16)
        Wf = torch.empty((w.Dff, w.D), device=x["Z"].device, dtype=torch.float32)
        lib = ttt.load_library()
        nbytes = lib.inplace_ttt_lm_workspace_size(w.T, w.Dff, w.D, w.Dm, w.C, w.k)
        ws = torch.empty(max(nbytes, 16), device=x["Z"].device, dtype=torch.uint8)
        return lambda: ttt.inplace_ttt_lm_chunk_fwd(x["Z"], x["X"], x["Wc"], x["Wp"], x["W0"],
                                                    x["eta"], C=w.C, O=O, W_out=Wf, workspace=ws)
    if w.kind == "inplace":
        O = torch.empty((w.T, w.D), device=x["Z"].device, dtype=torch.bfloat16)
        Wf = torch.empty((w.Dff, w.D), device=x["Z"].device, dtype=torch.float32)
        lib = ttt.load_library()
        nbytes = lib.inplace_ttt_workspace_size(w.T, w.Dff, w.D, w.C)
        ws = torch.empty(max(nbytes, 16), device=x["Z"].device, dtype=torch.uint8)
        return lambda: ttt.inplace_ttt_chunk_fwd(x["Z"], x["Vhat"], x["W0"], x["eta"], C=w.C,
                                                 O=O, W_out=Wf, workspace=ws)
    raise ValueError(w.kind)


def e2e_measure(w, x, steps: int, warmup: int):
    """Same metric through the public API from pinned HOST buffers: every step copies its inputs
    host->device, runs the operation and copies the result (O and the final state) back."""
    import torch

    import weight_linear_attention_ttt_b200 as ttt

    host = {k: v.cpu().pin_memory() for k, v in x.items() if torch.is_tensor(v)}
    dev = {k: torch.empty_like(v) for k, v in x.items() if torch.is_tensor(v)}
    scal = {k: v for k, v in x.items() if not torch.is_tensor(v)}
    if w.kind in ("inplace", "inplace_lm"):
        out_shapes = [((w.T, w.D), torch.bfloat16), ((w.Dff, w.D), torch.float32)]
    elif w.kind == "assoc_momentum":
        out_shapes = [((w.B, w.H, w.T, w.d), x["Q"].dtype), ((w.B, w.H, w.d, w.d), torch.float32),
                      ((w.B, w.H, w.d, w.d), torch.float32)]
    elif w.kind in ("assoc_bwd", "dual_bwd", "dual_seg_bwd"):
        out_shapes = [((w.B, w.H, w.T, w.d), x["Q"].dtype)] * 3 + [
            ((w.B, w.H, w.T), torch.float32), ((w.B, w.H, w.d, w.d), torch.float32)]
    else:
        out_shapes = [((w.B, w.H, w.T, w.d), x["Q"].dtype), ((w.B, w.H, w.d, w.d), torch.float32)]
    outs_h = [torch.empty(s, dtype=dt).pin_memory() for s, dt in out_shapes]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    xd = dict(dev, **scal)
    if not w.kind.startswith("inplace") and x.get("eta") is None:
        xd["eta"] = None
    call = make_call(w, xd)

    def step():
        for k in host:
            dev[k].copy_(host[k], non_blocking=True)
        outs = call()
        for h, d in zip(outs_h, outs):
            h.copy_(d, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    return ms, h2d, d2h


STREAM_KINDS = ("dual", "dual_seg", "assoc", "assoc_bwd", "assoc_momentum", "dual_bwd",
                "dual_seg_bwd")
ORACLE_ROUTINE = {"dual": "dual-form per-chunk loop", "dual_seg": "dual-form per-chunk loop",
                  "assoc": "sequential recurrence", "assoc_momentum": "momentum recurrence",
                  "dual_bwd": "dual-form chunk adjoint sweeps",
                  "dual_seg_bwd": "dual-form chunk adjoint sweeps",
                  "assoc_bwd": "adjoint sweeps of the recurrence"}


def host_cores() -> int:
    """Cores this process may run on (its affinity mask)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _pool_init(root: str):
    # one BLAS thread per worker: the workers already occupy every core
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"
    if root not in sys.path:
        sys.path.insert(0, root)


def _oracle_streams_task(kind: str, C: int, eta_const, beta, arrays: dict) -> int:
    """Runs the fp64 oracle over a group of whole (b,h) streams in a pool worker; returns the
    token-head count processed. `arrays` holds [n, tokens, d] slices (and [n, tokens] rates)."""
    from oracle import ttt_oracle as orc

    Q, K, V = arrays["Q"], arrays["K"], arrays["V"]
    n, ncol = Q.shape[0], Q.shape[1]
    for i in range(n):
        e = eta_const if arrays.get("eta") is None else arrays["eta"][i]
        if kind in ("dual", "dual_seg"):
            orc.dual_form_stream(Q[i], K[i], V[i], e, arrays["W0"][i], C)
        elif kind == "assoc_momentum":
            orc.assoc_momentum_stream(Q[i], K[i], V[i], e, beta, None, None)
        elif kind in ("dual_bwd", "dual_seg_bwd"):
            orc.dual_backward_stream(Q[i], K[i], V[i], e, arrays["W0"][i], arrays["dO"][i],
                                     arrays["G"][i], C)
        elif kind == "assoc_bwd":
            orc.assoc_backward_stream(Q[i], K[i], V[i], e, None, arrays["dO"][i],
                                      arrays["G"][i])
        else:
            orc.assoc_recurrence_stream(Q[i], K[i], V[i], e, None)
    return n * ncol


_POOL = {}


def close_oracle_pools():
    for p in _POOL.values():
        p.close()
        p.join()
    _POOL.clear()


def oracle_pool(cores: int):
    """A process pool for the oracle, started with spawn (a forked child of a process that has
    used CUDA can hang)."""
    import multiprocessing as mp

    if cores not in _POOL:
        _POOL[cores] = mp.get_context("spawn").Pool(cores, initializer=_pool_init,
                                                    initargs=(ROOT,))
    return _POOL[cores]


def oracle_sample(w, x, budget_s: float, cursor: list):
    """Runs the fp64 oracle on a bounded sample of the workload on the host's cores; returns
    (tokens, seconds, cores, description).

    Stream workloads: whole (b,h) streams (a prefix of chunks when one stream exceeds the
    budget), in groups spread over a spawn-started process pool with one worker per core,
    timed by wall clock from the first submission to the last result; waves of groups are
    submitted until the budget is spent. In-Place: output-column subsets (columns are
    independent), one process with the BLAS library's own threads."""
    import numpy as np

    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp

    if w.kind in STREAM_KINDS:
        import torch

        cores = host_cores()
        streams = [(b, h) for b in range(w.B) for h in range(w.H)]
        ncol = w.T if w.kind in ("dual", "dual_seg", "dual_bwd", "dual_seg_bwd") else min(w.T, 4096)
        eta = x.get("eta")
        grad_key = "dS_out" if w.kind == "assoc_bwd" else "dW_out"

        def group(idx):
            sel = [streams[i % len(streams)] for i in idx]
            bi = torch.tensor([s[0] for s in sel])
            hi = torch.tensor([s[1] for s in sel])
            arr = {k: x[k][bi, hi, :ncol].double().numpy() for k in ("Q", "K", "V")}
            arr["eta"] = None if eta is None else eta[bi, hi, :ncol].double().numpy()
            arr["W0"] = x["W0"][bi, hi].double().numpy()
            if w.kind in ("assoc_bwd", "dual_bwd", "dual_seg_bwd"):
                arr["dO"] = x["dO"][bi, hi, :ncol].double().numpy()
                arr["G"] = x[grad_key][bi, hi].double().numpy()
            return arr

        pool = oracle_pool(cores)
        # size a group so that one takes roughly a tenth of the budget: time one stream first
        t0 = time.perf_counter()
        _oracle_streams_task(w.kind, w.C, w.eta_const, inp.MOMENTUM_BETA,
                             group([cursor[0] % len(streams)]))
        per_stream = max(1e-4, time.perf_counter() - t0)
        per_group = max(1, min(len(streams), int(0.1 * budget_s / per_stream)))
        tok, waves = 0, 0
        t0 = time.perf_counter()
        while True:
            jobs = []
            for _ in range(cores):
                idx = list(range(cursor[0], cursor[0] + per_group))
                cursor[0] += per_group
                jobs.append(pool.apply_async(_oracle_streams_task,
                                             (w.kind, w.C, w.eta_const, inp.MOMENTUM_BETA,
                                              group(idx))))
            tok += sum(j.get() for j in jobs)
            waves += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        sec = time.perf_counter() - t0
        n_streams = tok // ncol
        desc = (f"{n_streams} (b,h) stream-runs x {ncol} tokens of the workload "
                f"({waves} wave(s) of {cores} groups of {per_group} streams), "
                f"{ORACLE_ROUTINE[w.kind]}, numpy fp64, {cores} worker processes")
        return tok / w.H, sec, cores, desc
    # In-Place: every 80th output column over all chunks (columns are independent)
    try:
        from threadpoolctl import threadpool_info

        blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        threads = max(blas) if blas else 1
    except Exception:
        threads = 1
    cols = np.arange(cursor[0] % 80, w.D, 80)
    cursor[0] += 1
    Z = x["Z"].float().cpu().numpy()
    W0 = x["W0"].float().cpu().numpy()[:, cols]
    if w.kind == "inplace_lm":
        Xh, Wc, Wp = (x[k].float().cpu().numpy() for k in ("X", "Wc", "Wp"))
        t0 = time.perf_counter()
        Vh = orc.lm_target(Xh, Wc, Wp[:, cols])
    else:
        Vh = x["Vhat"].float().cpu().numpy()[:, cols]
        t0 = time.perf_counter()
    orc.inplace_chunks(Z, Vh, W0, x["eta"], w.C)
    dt = time.perf_counter() - t0
    frac = len(cols) / w.D
    return w.T * frac, dt, threads, (f"{len(cols)} of {w.D} output columns over all "
                                     f"{w.T // w.C} chunks, numpy fp64 BLAS, {threads} threads")


# ----------------------------------------------------------------------------- arms
def config_of(w, world: int) -> dict:
    """The workload description both arms print (the reference arm times the same workload)."""
    from weight_linear_attention_ttt_b200 import metrics

    return {"workload": w.name, "kind": w.kind, "B": w.B, "H": w.H, "T": w.T, "d": w.d,
            "C": w.C, "tokens_per_step_per_gpu": metrics.algorithmic(w)["tokens"],
            "l2": "flushed (512 MiB write) before every timed step",
            "parallelism": f"dp{world} (independent streams per rank)"}


def run_reference(args, w, rank, world):
    """The oracle as the reference arm, on rank 0's host cores."""
    import torch

    from weight_linear_attention_ttt_b200 import inputs as inp

    if rank != 0:
        return 0
    x = inp.make_inputs(w, "cpu")
    cursor = [0]
    per_step_budget = max(0.05, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, x, per_step_budget, cursor)
    tok_total, sec_total, threads, desc = 0.0, 0.0, 1, ""
    for _ in range(args.steps):
        tok, sec, threads, desc = oracle_sample(w, x, per_step_budget, cursor)
        tok_total += tok
        sec_total += sec
    value = tok_total / sec_total
    ms = 1e3 * sec_total / args.steps
    line = {"impl": "reference", "metric": metric_of(w), "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import weight_linear_attention_ttt_b200 as ttt
    from weight_linear_attention_ttt_b200 import inputs as inp
    from weight_linear_attention_ttt_b200 import metrics
    from weight_linear_attention_ttt_b200.shard import max_over_ranks

    dev = torch.device("cuda", local_rank)
    ttt.load_library()
    for kv in args.tuning:
        k, v = kv.split("=")
        ttt.set_tuning(k, int(v))
    x = inp.make_inputs(w, dev, seed=w.seed + 7919 * rank)
    step = make_call(w, x)
    # 512 MiB write between timed steps: flushes the 126 MB L2, and runs long enough that the
    # host's argument marshalling and launch of the next call finish before it does
    flush = torch.empty(512 << 20, device=dev, dtype=torch.uint8)
    algo = metrics.algorithmic(w)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = ttt.launch_count()
    with ClockSampler(local_rank) as clk:
        for a, b in ev:
            flush.zero_()
            a.record()
            step()
            b.record()
        torch.cuda.synchronize()
    launches = ttt.launch_count() - n0
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
    ms_per_step = total_ms / args.steps
    value = world * algo["tokens"] * args.steps / (total_ms / 1e3)
    assert ttt.read_device_error() == 0, "a bounded device wait gave up during the bench"

    # end to end from host buffers, same metric
    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms, h2d, d2h = e2e_measure(w, x, e2e_steps, 2)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    e2e_value = world * algo["tokens"] / (e2e_ms / 1e3)

    pk, pk_kind = peaks()
    kname, ksrc = DOMINANT_KERNEL[w.kind]
    if w.kind == "dual" and ttt.get_tuning("dual_kernel") == 5:   # the TMEM-state kernel
        kname, ksrc = "dual_gram_kernel", "dual_gram.cu"
    if w.kind == "dual" and ttt.get_tuning("dual_kernel") == 6:   # the register-state Gram kernel
        kname, ksrc = "dual_rgram_kernel", "dual_rgram.cu"
    if w.kind == "assoc_momentum" and ttt.get_tuning("momentum_form") == 1:   # two-pass form
        kname, ksrc = "assoc_chunk_kernel", "assoc_scan.cu"
    if w.kind == "assoc_bwd" and ttt.get_tuning("assoc_bwd_form") == 1:   # separate passes
        kname, ksrc = "assoc_chunk_kernel", "assoc_scan.cu"
    if w.kind in ("dual_bwd", "dual_seg_bwd") and ttt.get_tuning("dual_bwd_form") in (1, 2):
        kname, ksrc = "dual_bwd_kernel", "dual_bwd.cu"   # the warp-MMA reverse sweep
    launches_per_step = launches / args.steps
    # the roofline is the slower of the flops at the tensor peak and the bytes at HBM bandwidth
    t_flops = algo["flops"] / (pk["bf16_tflops"] * 1e12)
    t_bytes = algo["bytes"] / (pk["hbm_gbs"] * 1e9)
    if t_flops > t_bytes:
        achieved = algo["flops"] / (ms_per_step / 1e3) / 1e12
        peak = pk["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak}
    else:
        achieved = algo["bytes"] / (ms_per_step / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak}
    roof["roofline_us"] = 1e6 * max(t_flops, t_bytes)
    sha = kernel_source_sha(ksrc)
    traffic, traffic_scope = measured_traffic(w.name, kname, sha)
    roof.update({"traffic": traffic, "traffic_scope": traffic_scope, "kernel": kname,
                 "peak_source": f"{pk_kind} (MEASURED_PEAKS.json)" if pk_kind == "measured"
                 else "fallback", "launches_per_step": launches_per_step,
                 "kernel_source_sha": sha,
                 "duration_us": 1e3 * ms_per_step
                 if w.kind in ("dual", "dual_bwd") and launches_per_step <= 1.0 else None})

    line = {"metric": metric_of(w), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": dict(config_of(w, world), **({"tuning": args.tuning} if args.tuning else {})),
            "roofline": roof, "clocks": clk.summary(), "gpu_launches": launches,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cursor = [0]
        budget = args.cpu_budget
        tok, sec, threads, desc = oracle_sample(w, {k: (v.cpu() if torch.is_tensor(v) else v)
                                                    for k, v in x.items()}, budget, cursor)
        line["cpu_baseline"] = {"value": tok / sec, "unit": "tokens/s", "cores": threads,
                                "kind": "oracle", "sample": desc, "seconds": sec}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tuning", action="append", default=[],
                    help="kernel-variant choice for comparisons, e.g. dual_kernel=1 (see "
                         "ttt_set_tuning in include/ttt.h)")
    ap.add_argument("--override", action="append", default=[],
                    help="shape override of the workload for reduced profiling cases, e.g. T=8192")
    args = ap.parse_args(argv)
    from weight_linear_attention_ttt_b200 import inputs as inp

    w = inp.WORKLOADS[args.workload]
    if args.override:
        import dataclasses

        w = dataclasses.replace(w, **{k: int(v) for k, v in (o.split("=") for o in args.override)})
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        try:
            return run_reference(args, w, rank, world)
        finally:
            close_oracle_pools()
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, w, rank, world, local_rank)
    finally:
        close_oracle_pools()
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
