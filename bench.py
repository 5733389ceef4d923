#!/usr/bin/env python3
"""Benchmark of the KDA forward scan (and the fused mShortConv -> KDA path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libkda|reference]
                    [--workload NAME] [--extra] [--no-cpu-baseline]

One JSON line on stdout (rank 0).  A step is one kda_forward call over one batch of
the workload (inputs resident in HBM).  Timing: W untimed warm-up steps, then K steps
bracketed by a barrier and torch.cuda.synchronize() on both sides, a CUDA event on the
launching stream after every step; the step time is the median over the K steps, max
over ranks.  The inputs (672 MB per step for the video clip) are larger than the
126 MB L2, so no flush is needed between steps.  Per-kernel times come from a separate
pass after the timed region.  The default run also times the other forward workloads
(image stream, fused conv + scan, long video) and reports them under extra_workloads.

Multi-GPU (torchrun): the ranks run the sequence-parallel forward of one stream of
N x T tokens, rank r holding the r-th T-token shard (weak scaling: per-rank work is
fixed); the exchange is one NCCL all-gather of the shards' affine maps per step.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0 only).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from linear_attention_sequence_mshortconv_b200 import inputs as W  # noqa: E402

METRIC = "KDA fwd Mtokens/s (H=16,d=128,T≈32k) and % of B200 roofline"
UNIT = "Mtokens/s"
DEFAULT_WORKLOAD = W.VIDEO_CLIP.name
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------------

def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def algorithmic_bytes(w: W.Workload) -> int:
    """Bytes a single pass must move: q, k, v, g read and o written at the run dtype,
    beta read, plus the fp32 final state written."""
    es = torch.tensor([], dtype=w.dtype).element_size()
    per_tok_head = 5 * w.D * es + es
    state = w.B * w.H * w.D * w.D * 4
    return w.B * w.T * w.H * per_tok_head + state


def conv_fmas(w: W.Workload) -> int:
    """Multiply-adds of mShortConv per step: taps x channels x tokens, for q, k and v."""
    taps = {0: w.Kt, 1: 9, 2: 27}
    C = w.H * w.D
    n = 0
    for (mod, _start, Fr, Hh, Wd, _ws) in w.segments:
        toks = Wd if mod == 0 else (Hh * Wd if mod == 1 else Fr * Hh * Wd)
        n += toks * taps[mod] * C
    return 3 * w.B * n


_FMA_RATE = None


def conv_alu_roofline(w: W.Workload, conv_ms: float):
    """The conv's plain-ALU term: its multiply-adds per second against this GPU's fp32
    FMA rate measured by the library's probe kernel."""
    global _FMA_RATE
    from linear_attention_sequence_mshortconv_b200 import kda
    if _FMA_RATE is None:
        _FMA_RATE = kda.fma_probe()
    achieved = conv_fmas(w) / (conv_ms * 1e-3)
    return {"bound": "alu", "achieved": achieved / 1e12, "peak": _FMA_RATE / 1e12, "unit": "TFMA/s",
            "frac": achieved / _FMA_RATE, "peak_source": "measured (kda_fma_probe)",
            "fmas_per_step": conv_fmas(w)}


def traffic_record(workload: str):
    """DRAM bytes (read + write) of one whole forward call of the workload from the
    committed ncu summary, if it was taken on the current source of the scan kernel
    (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            recs = json.load(f)
    except (OSError, ValueError):
        return None
    rec = recs.get(workload)
    if not rec:
        return None
    src = os.path.join(ROOT, rec.get("source", ""))
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    if sha != rec.get("source_sha256"):
        return None
    return rec.get("dram_bytes_per_step")


class ClockSampler:
    """Polls NVML (SM clock and throttle reasons) in a thread during the timed region."""

    REASONS = {  # NVML clocks-event reason bits
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ----------------------------------------------------------------------------------

def oracle_sample_tokens(w: W.Workload, target_s: float, threads: int) -> int:
    """Prefix length (all heads, batch row 0) that takes about target_s on the oracle."""
    from oracle import oracle as O
    probe = w.resized(B=1, T=min(w.T, 128), name="probe")
    inp = W.make_kda_inputs(probe)
    t0 = time.perf_counter()
    O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], want_o=True, nthreads=threads)
    dt = max(time.perf_counter() - t0, 1e-4)
    per_tok = dt / probe.T
    return int(max(64, min(w.T, target_s / per_tok)))


def time_oracle(w: W.Workload, T_s: int, threads: int):
    """Runs the oracle on the first T_s tokens (batch row 0, all heads); returns
    (seconds, tokens processed)."""
    from oracle import oracle as O
    sample = w.resized(B=1, T=T_s, name="sample")
    inp = W.make_kda_inputs(sample)
    t0 = time.perf_counter()
    O.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], want_o=True, nthreads=threads)
    return time.perf_counter() - t0, T_s


def cpu_baseline(w: W.Workload, target_s: float = 12.0):
    from oracle import oracle as O
    threads = O.default_threads()
    T_s = oracle_sample_tokens(w, target_s, threads)
    secs, toks = time_oracle(w, T_s, threads)
    return {"value": toks / secs / 1e6, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"fp64 token loop, first {T_s} of {w.T} tokens of batch row 0, all {w.H} "
                      f"heads ({secs:.1f} s)"}


def run_reference(args, ws, rank, w: W.Workload):
    if rank != 0:
        return
    from oracle import oracle as O
    threads = O.default_threads()
    per_step = max(0.5, 90.0 / max(1, args.steps + args.warmup))
    T_s = oracle_sample_tokens(w, per_step, threads)
    for _ in range(args.warmup):
        time_oracle(w, T_s, threads)
    total, toks = 0.0, 0
    for _ in range(args.steps):
        s, n = time_oracle(w, T_s, threads)
        total += s
        toks += n
    value = toks / total / 1e6
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, ws),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"each step: fp64 token loop over the first {T_s} of "
                                       f"{w.T} tokens of batch row 0, all {w.H} heads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w: W.Workload, ws: int, sp: bool = False):
    par = "single GPU"
    if ws > 1:
        par = (f"sequence parallel x{ws}: one stream of {ws}x{w.T} tokens, rank r holds the r-th "
               f"{w.T}-token shard; one NCCL all-gather of the shard maps per step") if sp else f"replicas x{ws}"
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "d": w.D, "chunk": w.chunk,
            "fused_conv": w.fused, "parallelism": par,
            "l2": "inputs larger than L2 (no flush)" if algorithmic_bytes(w) > 126e6
                  else "L2 flushed between steps"}


# ----------------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------------

def make_sp_step(w: W.Workload, rank: int, world: int):
    """One step of the sequence-parallel forward of ONE stream of world * T tokens: rank r
    holds tokens [r*T, (r+1)*T) (its shard drawn from its own seed), runs the shard's state
    pass, takes part in the one NCCL all-gather of the shard maps, folds the earlier shards
    into its entry state and runs its output pass."""
    from linear_attention_sequence_mshortconv_b200 import sequence_parallel as SP
    dev = torch.device("cuda")
    inp = W.make_kda_inputs(W.dataclasses.replace(w, seed=w.seed + 1000 * rank), device=dev)
    box = {}

    def step():
        box["o"], box["S_T"] = SP.forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], chunk=w.chunk,
                                          o_dtype=w.dtype)
    step()
    torch.cuda.synchronize()
    return step, inp, box["o"], box["S_T"]


def make_step(w: W.Workload, rank: int):
    from linear_attention_sequence_mshortconv_b200 import kda
    dev = torch.device("cuda")
    wr = w if rank == 0 else W.dataclasses.replace(w, seed=w.seed + 1000 * rank)
    if w.fused:
        inp = W.make_fused_inputs(wr, device=dev)
        o = torch.empty((w.B, w.T, w.H, w.D), dtype=w.dtype, device=dev)
        S_T = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
        wsz = kda.mshortconv_workspace_size(w.B, w.T, w.H, w.D, w.dtype, w.chunk, o_dtype=w.dtype)
        ws = torch.empty(max(wsz, 1), dtype=torch.uint8, device=dev)

        def step():
            kda.mshortconv_kda_forward(inp["xq"], inp["xk"], inp["xv"], inp["segments"], w.Kt,
                                       inp["wq"], inp["wk"], inp["wv"], inp["g"], inp["beta"],
                                       chunk=w.chunk, o=o, S_T=S_T, workspace=ws)
        return step, inp, o, S_T
    inp = W.make_kda_inputs(wr, device=dev)
    o = torch.empty((w.B, w.T, w.H, w.D), dtype=w.dtype, device=dev)
    S_T = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
    wsz = kda.workspace_size(w.B, w.T, w.H, w.D, w.D, w.dtype, w.chunk)
    ws = torch.empty(max(wsz, 1), dtype=torch.uint8, device=dev)

    def step():
        kda.forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], chunk=w.chunk,
                    o=o, S_T=S_T, workspace=ws)
    return step, inp, o, S_T


def timed(step, K, ws):
    """K steps between a barrier + synchronize on both sides, with a CUDA event on the
    launching stream before the first step and after every step.  Returns (total ms,
    per-step ms list)."""
    barrier(ws)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    ev[0].record(s)
    for i in range(K):
        step()
        ev[i + 1].record(s)
    torch.cuda.synchronize()
    barrier(ws)
    return ev[0].elapsed_time(ev[K]), [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]


PROFILED = ("kda_generic", "kda_tc_state", "kda_tc_combine", "kda_tc_output", "kda_tc_output_first", "conv",
            "kda_sp_fold")


def kernel_profile(step, K):
    """Per-kernel device time from CUDA events the library records around its own launches,
    in a separate pass after the timed region (so the timed steps carry no extra events)."""
    from linear_attention_sequence_mshortconv_b200 import kda
    for name in PROFILED:
        kda.profile_collect(name)
    kda.profile_enable(True)
    for _ in range(K):
        step()
    torch.cuda.synchronize()
    kda.profile_enable(False)
    prof = {}
    for name in PROFILED:
        r = kda.profile_collect(name)
        if r and r[1] > 0:
            prof[name] = {"ms_per_step": r[0] / K, "launches_per_step": r[1] / K, "ms_per_launch": r[0] / r[1]}
    return prof


def step_roofline(w: W.Workload, ms_step: float, peaks, peak_kind, prof=None):
    """The forward call's roofline: its algorithmic bytes over the median step time against
    the measured HBM copy bandwidth (the bound), and the chunk method's useful tensor FLOPs
    against the measured bf16 GEMM rate.  Per-kernel shares of the step under "kernels"."""
    alg = algorithmic_bytes(w)
    achieved = alg / (ms_step * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": traffic_record(w.name), "algorithmic_bytes_per_step": alg, "peak_source": peak_kind,
            "scope": "whole forward call (every kernel of the step)"}
    if w.D == 128 and w.dtype != torch.float32:
        flops = (5 * 64 * w.D + 6 * w.D * w.D) * w.tokens * w.H
        tf = flops / (ms_step * 1e-3) / 1e12
        bf = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
        roof["tensor_step"] = {"achieved": tf, "peak": bf, "unit": "TFLOP/s", "frac": tf / bf, "flops_per_step": flops}
    if prof:
        roof["kernels"] = {n: {**v, "share_of_step": v["ms_per_step"] / ms_step} for n, v in prof.items()}
    return roof


def e2e_measure_sp(w: W.Workload, K: int, ws: int, rank: int):
    """The sequence-parallel step through the public API with host buffers: every step
    uploads this rank's shard from pinned host memory, runs the sharded forward (with its
    all-gather) and reads o and S_T back; max over ranks."""
    from linear_attention_sequence_mshortconv_b200 import sequence_parallel as SP
    host = W.make_kda_inputs(W.dataclasses.replace(w, seed=w.seed + 1000 * rank), device="cpu")
    host = {k: v.pin_memory() for k, v in host.items() if isinstance(v, torch.Tensor)}
    dv = {k: torch.empty_like(v, device="cuda") for k, v in host.items()}
    o_h = torch.empty((w.B, w.T, w.H, w.D), dtype=w.dtype).pin_memory()
    S_h = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * 4

    def step():
        for k_, v in host.items():
            dv[k_].copy_(v, non_blocking=True)
        o, S_T = SP.forward(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], chunk=w.chunk, o_dtype=w.dtype)
        o_h.copy_(o, non_blocking=True)
        S_h.copy_(S_T, non_blocking=True)
    step()
    total, per = timed(step, K, ws)
    ms = max_over_ranks(statistics.median(per), ws)
    return {"value": ws * w.tokens / (ms * 1e-3) / 1e6, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "pipelined": "no (copies, call and read-back in order)"}


def e2e_measure(w: W.Workload, K: int, ws: int, rank: int, sp: bool = False):
    """Same metric through the public API with HOST buffers: every step copies its inputs
    from pinned host memory, runs the call and reads o and S_T back.  Steps are
    pipelined over three streams with two device buffer sets: the upload of step n+1
    runs while step n computes and while step n's result is read back (the link carries
    the two directions at once).  The timed region runs from before the first upload to
    after the last read-back."""
    from linear_attention_sequence_mshortconv_b200 import kda
    if sp:
        return e2e_measure_sp(w, K, ws, rank)
    dev = torch.device("cuda")
    host = W.make_kda_inputs(w, device="cpu") if not w.fused else None
    if host is None:
        return None
    host = {k: v.pin_memory() for k, v in host.items() if isinstance(v, torch.Tensor)}
    dv = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    o = [torch.empty((w.B, w.T, w.H, w.D), dtype=w.dtype, device=dev) for _ in range(2)]
    S_T = [torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev) for _ in range(2)]
    o_h = torch.empty_like(o[0], device="cpu").pin_memory()
    S_h = torch.empty_like(S_T[0], device="cpu").pin_memory()
    wsz = kda.workspace_size(w.B, w.T, w.H, w.D, w.D, w.dtype, w.chunk)
    wbuf = torch.empty(max(wsz, 1), dtype=torch.uint8, device=dev)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o[0].numel() * o[0].element_size() + S_T[0].numel() * 4
    s_c = torch.cuda.current_stream()
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    up_done = [ev(), ev()]      # buffer set b holds step n's inputs
    comp_done = [ev(), ev()]    # step n's compute has read set b and written o[b]
    down_done = [ev(), ev()]    # o[b], S_T[b] have been read back

    def run(K_):
        def upload(n):
            b = n % 2
            if n >= 2:
                s_up.wait_event(comp_done[b])
            with torch.cuda.stream(s_up):
                for k_, v in host.items():
                    dv[b][k_].copy_(v, non_blocking=True)
            up_done[b].record(s_up)

        upload(0)
        for n in range(K_):
            b = n % 2
            if n + 1 < K_:
                upload(n + 1)
            s_c.wait_event(up_done[b])
            if n >= 2:
                s_c.wait_event(down_done[b])
            d = dv[b]
            kda.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], chunk=w.chunk, o=o[b], S_T=S_T[b],
                        workspace=wbuf, stream=s_c)
            comp_done[b].record(s_c)
            s_down.wait_event(comp_done[b])
            with torch.cuda.stream(s_down):
                o_h.copy_(o[b], non_blocking=True)
                S_h.copy_(S_T[b], non_blocking=True)
            down_done[b].record(s_down)
        s_c.wait_event(down_done[(K_ - 1) % 2])

    run(2)
    torch.cuda.synchronize()
    barrier(ws)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_c)
    run(K)
    e.record(s_c)
    torch.cuda.synchronize()
    barrier(ws)
    ms = max_over_ranks(a.elapsed_time(e), ws)
    return {"value": ws * w.tokens / (ms / K * 1e-3) / 1e6, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / K,
            "pipelined": "upload of step n+1 overlaps compute and read-back of step n"}


def forward_record(w: W.Workload, K: int, peaks, peak_kind):
    """One other forward workload, device-timed like the headline (median of K steps), with
    its call-level roofline and per-kernel profile (and the conv's ALU term when fused)."""
    st, _, _, _ = make_step(w, 0)
    for _ in range(3):
        st()
    total, per = timed(st, K, 1)
    m = statistics.median(per)
    prof = kernel_profile(st, max(3, K // 4))
    rec = {"workload": w.name, "ms_per_step": m, "ms_per_step_mean": total / K, "steps": K,
           "value": w.tokens / (m * 1e-3) / 1e6, "unit": UNIT,
           "roofline": step_roofline(w, m, peaks, peak_kind, prof)}
    if w.fused and "conv" in prof:
        rec["conv_alu"] = conv_alu_roofline(w, prof["conv"]["ms_per_step"])
    torch.cuda.synchronize()
    return rec


def run_gpu(args, ws, rank, local, w: W.Workload):
    from linear_attention_sequence_mshortconv_b200 import build as libbuild
    from linear_attention_sequence_mshortconv_b200 import kda
    if rank == 0:
        libbuild.build()
    barrier(ws)
    kda.load_library()
    sp = ws > 1 and not w.fused
    step, inp, o, S_T = make_sp_step(w, rank, ws) if sp else make_step(w, rank)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if not torch.isfinite(o.float()).all():
        raise RuntimeError("non-finite output")

    launches0 = kda.kernel_launches()
    sampler = ClockSampler(local)
    with sampler:
        total, per = timed(step, args.steps, ws)
    launches = kda.kernel_launches() - launches0
    ms_med = max_over_ranks(statistics.median(per), ws)
    ms_mean = max_over_ranks(total / args.steps, ws)
    value = ws * w.tokens / (ms_med * 1e-3) / 1e6
    peaks, peak_kind = read_peaks()
    prof = kernel_profile(step, max(3, args.steps // 4))
    roof = step_roofline(w, ms_med, peaks, peak_kind, prof)
    if not w.fused:
        P_, L_ = kda.forward_plan(w.B, w.T, w.H, w.D, w.D, w.dtype, w.chunk)
        roof["split"] = {"segments": P_, "chunks_per_segment": L_}

    e2e = None if args.quick else e2e_measure(w, max(3, min(args.steps, 10)), ws, rank, sp=sp)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not args.quick:
        cpu = cpu_baseline(w)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_med, "ms_per_step_mean": ms_mean,
            "timing": "median of the per-step CUDA-event times (value uses it); mean = total / steps",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": workload_config(w, ws, sp), "roofline": roof, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": launches, "clocks": sampler.summary()}
    if rank == 0 and not args.quick:
        # the other forward configurations of the workload set, each on its own line entry
        others = [x for x in (W.IMAGE_STREAM, W.FUSED_MIXED, W.LONG_VIDEO) if x.name != w.name and not args.tokens]
        line["extra_workloads"] = [forward_record(x, max(20, args.steps), peaks, peak_kind) for x in others]
    if args.extra and rank == 0:
        extra = line.setdefault("extra_workloads", [])
        # the headline workload with the output side of Eq. 15 fused (Sigmoid(gate) *
        # RMSNorm(readout)); its extra bytes are the gate read
        if not w.fused:
            inp_g = W.make_kda_inputs(w, device="cuda")
            gen = torch.Generator().manual_seed(7)
            gate = torch.randn(w.B, w.T, w.H, w.D, generator=gen).to(w.dtype).cuda()
            gamma = (0.5 + torch.rand(w.H, w.D, generator=gen)).cuda()
            og = torch.empty((w.B, w.T, w.H, w.D), dtype=w.dtype, device="cuda")
            Sg = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device="cuda")
            wsz = kda.workspace_size(w.B, w.T, w.H, w.D, w.D, w.dtype, w.chunk)
            wsb = torch.empty(max(wsz, 1), dtype=torch.uint8, device="cuda")

            def gstep():
                kda.forward_gated(inp_g["q"], inp_g["k"], inp_g["v"], inp_g["g"], inp_g["beta"], gate, gamma,
                                  1e-6, chunk=w.chunk, o=og, S_T=Sg, workspace=wsb)
            for _ in range(3):
                gstep()
            k_g = max(3, args.steps // 4)
            mg = timed(gstep, k_g, 1)[0] / k_g
            gbytes = algorithmic_bytes(w) + w.B * w.T * w.H * w.D * torch.tensor([], dtype=w.dtype).element_size()
            extra.append({"workload": w.name + "_gated_output", "ms_per_step": mg,
                          "value": w.tokens / (mg * 1e-3) / 1e6, "unit": UNIT,
                          "alg_GBps": gbytes / (mg * 1e-3) / 1e9,
                          "epilogue": "Sigmoid(gate) * RMSNorm(S_t^T q_t), fused in the output stage"})
        # one rank's local work in a sequence-parallel run: the last of 8 time shards of
        # the long video row (its transition, the prefix over the 7 earlier shards' maps,
        # its output pass); the all-gather of the maps (2 MiB per rank) is not included
        if not w.fused:
            R = 8
            sw = W.LONG_VIDEO.resized(T=W.LONG_VIDEO.T // R, name="long_video_shard_8_of_8")
            si = W.make_kda_inputs(sw, device="cuda")
            wss = kda.sp_workspace(si["q"], sw.chunk)
            MN_all = torch.zeros((R, sw.B, sw.H, 2, sw.D, sw.D), dtype=torch.float32, device="cuda")
            S_in = torch.empty((sw.B, sw.H, sw.D, sw.D), dtype=torch.float32, device="cuda")
            o_s = torch.empty((sw.B, sw.T, sw.H, sw.D), dtype=sw.dtype, device="cuda")
            S_s = torch.empty_like(S_in)
            kda.sp_transition(si["q"], si["k"], si["v"], si["g"], si["beta"], wss, chunk=sw.chunk, MN=MN_all[R - 1])
            MN_all[: R - 1].copy_(MN_all[R - 1].expand(R - 1, *MN_all.shape[1:]))

            def sstep():
                kda.sp_transition(si["q"], si["k"], si["v"], si["g"], si["beta"], wss, chunk=sw.chunk,
                                  MN=MN_all[R - 1])
                kda.sp_prefix(MN_all, R - 1, None, S_in=S_in)
                kda.sp_output(si["q"], si["k"], si["v"], si["g"], si["beta"], S_in, wss, chunk=sw.chunk,
                              o=o_s, S_T=S_s)
            for _ in range(3):
                sstep()
            k_s = max(3, args.steps // 4)
            kda.profile_enable(True)
            ms_s = timed(sstep, k_s, 1)[0] / k_s
            kda.profile_enable(False)
            kern = {}
            for name in ("kda_tc_state", "kda_sp_fold", "kda_tc_combine", "kda_tc_output"):
                r = kda.profile_collect(name)
                if r and r[1] > 0:
                    kern[name] = {"ms_per_step": r[0] / k_s, "launches_per_step": r[1] / k_s}
            extra.append({"workload": sw.name, "shard_tokens": sw.T, "ranks": R, "ms_per_step": ms_s,
                          "value": sw.T / (ms_s * 1e-3) / 1e6, "unit": UNIT + " (one rank's shard)",
                          "alg_GBps": algorithmic_bytes(sw) / (ms_s * 1e-3) / 1e9, "kernels": kern,
                          "excludes": "the all-gather of the ranks' maps"})
        # the backward of the headline workload (kda_backward: fp32 gradients of q, k, v,
        # g, beta, S0 for a random dL/do); algorithmic bytes: the forward's inputs and do
        # read once, the fp32 gradients written once
        if not w.fused:
            inp_b = W.make_kda_inputs(w, device="cuda")
            do_b = torch.randn(w.B, w.T, w.H, w.D, generator=torch.Generator().manual_seed(8)).to(w.dtype).cuda()
            f32 = dict(dtype=torch.float32, device="cuda")
            outs = (torch.empty((w.B, w.T, w.H, w.D), **f32), torch.empty((w.B, w.T, w.H, w.D), **f32),
                    torch.empty((w.B, w.T, w.H, w.D), **f32), torch.empty((w.B, w.T, w.H, w.D), **f32),
                    torch.empty((w.B, w.T, w.H), **f32), torch.empty((w.B, w.H, w.D, w.D), **f32))
            wsb_b = torch.empty(max(kda.backward_workspace_size(w.B, w.T, w.H, w.D, w.D), 1), dtype=torch.uint8,
                                device="cuda")

            def bstep():
                kda.backward(inp_b["q"], inp_b["k"], inp_b["v"], inp_b["g"], inp_b["beta"], do_b,
                             workspace=wsb_b, out=outs)
            for _ in range(3):
                bstep()
            k_b = 5
            mb = timed(bstep, k_b, 1)[0] / k_b
            esz = torch.tensor([], dtype=w.dtype).element_size()
            bbytes = algorithmic_bytes(w) + w.B * w.T * w.H * (4 * w.D * 4 + 4)
            # the kernel's fp32 matrix-product multiply-adds per (32-token chunk C, 16 value
            # columns Vc, key width D): forward sweep C^2 D + 2 C D Vc + C^2 Vc; reverse sweep
            # (T and Kd read back) 5 C^2 D + 7 C D Vc + 5 C^2 Vc + 2 C^3.  They run as 3xTF32 warp MMAs (three TF32
            # products per fp32 product), so the bound is the TF32 tensor rate: the measured
            # bf16 GEMM peak x the nominal TF32/bf16 ratio (1.1 / 2.25 PFLOP/s), divided by 3.
            C_, Vc_, D_ = 32, 16, w.D
            fma_chunk = 6 * C_ * C_ * D_ + 9 * C_ * D_ * Vc_ + 6 * C_ * C_ * Vc_ + 2 * C_ ** 3
            fmas = fma_chunk * w.B * w.H * (w.D // Vc_) * ((w.T + C_ - 1) // C_)
            peak_tf = float(peaks.get("bf16_tflops", PEAKS_FALLBACK.get("bf16_tflops", 1590.0))) * (1.1 / 2.25) / 3
            ach_tf = 2 * fmas / (mb * 1e-3) / 1e12
            extra.append({"workload": w.name + "_backward", "ms_per_step": mb,
                          "value": w.tokens / (mb * 1e-3) / 1e6, "unit": UNIT,
                          "alg_GBps": bbytes / (mb * 1e-3) / 1e9, "alg_bytes": bbytes,
                          "roofline": {"bound": "tensor", "achieved": ach_tf, "peak": peak_tf, "unit": "TFLOP/s",
                                       "frac": ach_tf / peak_tf, "flops_per_step": 2 * fmas,
                                       "peak_source": "measured bf16 GEMM x nominal TF32/bf16 ratio / 3 (3xTF32)"},
                          "path": "3xTF32 warp MMAs for every matrix product, fp32 elsewhere; one CTA per "
                                  "(b, h, 16 value columns)"})
        # mShortConv backward on the fused workload's stream (one tensor, x_q: dx and the
        # three modalities' weight gradients); bound: plain ALU (its multiply-adds are the
        # forward's twice over: dx and dw)
        fw = W.FUSED_MIXED
        fin = W.make_fused_inputs(fw, device="cuda")
        dy_c = torch.randn(fw.B, fw.T, fw.H * fw.D, generator=torch.Generator().manual_seed(9)).to(fw.dtype).cuda()
        wq = fin["wq"]

        def cstep():
            kda.mshortconv_backward(fin["xq"], dy_c, fin["segments"], fw.Kt, wq[0], wq[1], wq[2])
        for _ in range(3):
            cstep()
        k_c = 5
        mc = timed(cstep, k_c, 1)[0] / k_c
        cf = 2 * conv_fmas(fw) // 3
        rate = kda.fma_probe()
        extra.append({"workload": fw.name + "_conv_backward_xq", "ms_per_step": mc,
                      "roofline": {"bound": "alu", "achieved": cf / (mc * 1e-3) / 1e12, "peak": rate / 1e12,
                                   "unit": "TFMA/s", "frac": cf / (mc * 1e-3) / rate, "fmas_per_step": cf,
                                   "peak_source": "kda_fma_probe on this GPU"},
                      "path": "shared-memory tiles (8 rows x 16 positions + halo, 64 channels), register windows; dw one atomic per (channel, tap) per tile"})
        # backward of the whole fused path on the fused workload (kda_mshortconv_backward)
        fb_do = torch.randn(fw.B, fw.T, fw.H, fw.D, generator=torch.Generator().manual_seed(10)).to(fw.dtype).cuda()
        fb_ws = torch.empty(max(1, kda.mshortconv_kda_backward_workspace_size(fw.B, fw.T, fw.H, fw.D, fw.dtype)),
                            dtype=torch.uint8, device="cuda")

        def fbstep():
            kda.mshortconv_kda_backward(fin["xq"], fin["xk"], fin["xv"], fin["segments"], fw.Kt, fin["wq"], fin["wk"],
                                        fin["wv"], fin["g"], fin["beta"], fb_do, workspace=fb_ws)
        for _ in range(2):
            fbstep()
        mf = timed(fbstep, 3, 1)[0] / 3
        extra.append({"workload": fw.name + "_backward", "ms_per_step": mf,
                      "value": fw.tokens / (mf * 1e-3) / 1e6, "unit": UNIT,
                      "path": "fp32 conv recompute, per-head norm, kda_backward, norm and conv backward"})
        line["extra_workloads"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_part(args, w: W.Workload):
    """One other call on the workload, device-timed: the scan's backward (kda_backward on
    the workload's q, k, v, g, beta and a random dL/do) or the conv backward of x_q (a
    workload with a conv).  Not the benchmark step; used to profile those kernels."""
    from linear_attention_sequence_mshortconv_b200 import build as libbuild
    from linear_attention_sequence_mshortconv_b200 import kda
    libbuild.build()
    kda.load_library()
    gen = torch.Generator().manual_seed(11)
    if args.part == "backward":
        inp = W.make_kda_inputs(w, device="cuda")
        do = torch.randn(w.B, w.T, w.H, w.D, generator=gen).to(w.dtype).cuda()
        wsb = torch.empty(max(1, kda.backward_workspace_size(w.B, w.T, w.H, w.D, w.D)), dtype=torch.uint8,
                          device="cuda")

        def step():
            kda.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], do, workspace=wsb)
    else:
        fin = W.make_fused_inputs(w, device="cuda")
        dy = torch.randn(w.B, w.T, w.H * w.D, generator=gen).to(w.dtype).cuda()

        def step():
            kda.mshortconv_backward(fin["xq"], dy, fin["segments"], w.Kt, *fin["wq"])
    for _ in range(max(1, args.warmup)):
        step()
    ms = timed(step, args.steps, 1)[0] / args.steps
    print(json.dumps({"part": args.part, "workload": w.name, "ms_per_step": ms, "steps": args.steps,
                      "tokens": w.tokens}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libkda", choices=["libkda", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.BY_NAME))
    ap.add_argument("--extra", action="store_true", help="also time the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true",
                    help="device timing only: no end-to-end leg, no CPU baseline (for profiling)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload on its first N tokens (smaller profiling cases)")
    ap.add_argument("--part", default="forward", choices=["forward", "backward", "conv_backward"],
                    help="time one other call on the workload instead of the forward step "
                         "(single GPU; prints its own JSON line; for profiling)")
    args = ap.parse_args()
    ws, rank, local = dist_setup()
    w = W.BY_NAME[args.workload]
    if args.tokens:
        w = w.resized(T=args.tokens, name=f"{w.name}_first{args.tokens}")
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank, w)
        elif args.part != "forward":
            run_part(args, w)
        else:
            run_gpu(args, ws, rank, local, w)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
