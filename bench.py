"""Throughput of the S6 selective scan on B200 -- one JSON line on rank 0.

A step is one pass of the hot path over one batch: the fused causal conv4 +
SiLU + selective scan + SiLU(z) gate + h_final of the long-sequence workload
(Bt16 L8192 d1536 N16, bf16 I/O, float32 state, simplified dt*B write), i.e.
one s6_conv_scan_fwd launch over 201M (b, t, channel) elements.  Inputs
(1.2 GB per step) are larger than L2, so no flush is needed between steps.

metric: Gelem/s = Bt*L*d_inner / time.  value: whole job (all ranks).
Also reported: the roofline of the dominant kernel (MUFU ex2: N = 16
exponentials per element; HBM alongside), the oracle on the host cores
(cpu_baseline), the same metric end to end from pinned host buffers (e2e,
pipelined over batch chunks), and rows for the rest of the path, each with its
own roofline: the other workloads of the pages (Mamba-mini, wide, one long
prompt), random A_log, the streaming-decode step, the decode block, the
constant-decay cell, the standalone conv, a chunked prefill, the two
backward passes and a training step (forward keeping checkpoints, backward
from them).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: torchrun ... bench.py --gpus N; each rank scans its own batch (weak
scaling, no data-path collective); the time is the max over ranks.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import s6_inputs as SI  # noqa: E402

METRIC = "selective-scan Gelem/s (B·L·d_inner) and % of HBM/MUFU-ex2 roofline"
WORKLOAD = "long_seq"
SMS = 148
MUFU_PER_SM_CLK = 16  # ex2 results per SM per clock (special-function unit)
HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0  # dense bf16 GEMM, burst


def peaks():
    p = {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": BF16_FALLBACK_TFLOPS, "sm_max_mhz": 1965.0,
         "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        p.update(hbm_gbs=float(m["hbm_gbs"]), bf16_tflops=float(m.get("bf16_tflops", BF16_FALLBACK_TFLOPS)),
                 sm_max_mhz=float(m.get("sm_max_mhz", 1965.0)), source="measured")
    return p


def algorithmic_bytes_per_elem(cfg, gate=True):
    """x, dt, z read + y written per element, B and C rows per token shared by d channels."""
    s = 2 if cfg["io"] == "bf16" else 4
    per = (3 if gate else 2) * s + s
    return per + 2 * cfg["N"] * s / cfg["d"]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock, power and throttle reasons sampled in a background thread through
    NVML (about every 2 ms, so that a timed region of a few tens of ms still gets
    a record of its own); nvidia-smi polling when NVML is unavailable."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, period_ms: float = 2.0):
        self.dev = device_index
        self.period = period_ms / 1e3
        self.rows = []  # (sm_mhz, max_mhz, power_w, set of reason names, host time)
        self.thread = None
        self.proc = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        for bus in (f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0",
                    f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"):
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except pynvml.NVMLError:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._nvml_handle()
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.stop_flag = threading.Event()

            def loop():
                while not self.stop_flag.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1e3
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((float(sm), float(mx), pw, {k for k, b in bits.items() if rs & b},
                                          time.time()))
                    except pynvml.NVMLError:
                        pass
                    self.stop_flag.wait(self.period)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = "nvml"
        except Exception:  # no NVML: poll nvidia-smi instead
            self.thread = None
            fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                      "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                      "clocks_event_reasons.sw_power_cap")
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={fields}",
                                              "--format=csv,noheader,nounits", "-lms", "50"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
            except (OSError, ValueError):
                self.proc = None
        return self

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for line in out.splitlines():
                parts = [q.strip() for q in line.split(",")]
                if len(parts) >= 7:
                    try:
                        self.rows.append((float(parts[0]), float(parts[1]), float(parts[2]),
                                          {n for n, v in zip(self.NAMES, parts[3:7]) if v.lower() == "active"},
                                          None))
                    except ValueError:
                        pass

    def summary(self, window=None):
        """Summary of the samples taken inside `window` = (t0, t1) host seconds
        (all samples when None or when the source gives no times)."""
        rows = self.rows
        if window is not None:
            inside = [r for r in rows if r[4] is not None and window[0] <= r[4] <= window[1]]
            if inside:
                rows = inside
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples (NVML and nvidia-smi unavailable)"],
                    "samples": 0}
        mx = max(r[1] for r in rows)
        sm = [r[0] for r in rows]
        loaded = [v for v in sm if v > 0.5 * mx]
        reasons = sorted(set().union(*(r[3] for r in rows)))
        return {"sm_mhz": statistics.median(loaded or sm), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded), "source": self.source,
                "power_w_max": max(r[2] for r in rows), "sm_mhz_min": min(sm)}


# ------------------------------------------------------------------ helpers
def to_dev(a, device):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_pinned(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.pin_memory()


def kernel_source_sha():
    """Hash of the scan kernel's sources with comments and blank lines removed, so
    that an edit of a comment does not orphan the recorded capture."""
    h = hashlib.sha256()
    for f in ("s6_common.cuh", "s6_scan.cuh"):
        with open(os.path.join(ROOT, "selective_state_space_19_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the scan kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "s6_conv_scan_long_seq.md")
    if not os.path.exists(path):
        return None, None
    txt = open(path).read()
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    m_b = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", txt)
    if not (m_sha and m_b) or m_sha.group(1) != kernel_source_sha():
        return None, (m_sha.group(1) if m_sha else None)
    return float(m_b.group(1)), m_sha.group(1)


# ------------------------------------------------------------------ oracle leg
class OracleLeg:
    """The float64 oracle timed on the host cores over a bounded sample of the
    workload: a fixed, seeded set of (b, channel) pairs, each over the whole
    sequence.  The CPU-baseline leg and the reference arm time the same sample."""

    SAMPLE_PAIRS = 4096

    def __init__(self, inp, zoh, threads=None):
        self.inp, self.zoh = inp, zoh
        self.cores = threads or os.cpu_count() or 1
        rng = np.random.default_rng(99)
        n = min(self.SAMPLE_PAIRS, inp["Bt"] * inp["d"])
        self.ch = np.stack([rng.integers(0, inp["Bt"], n), rng.integers(0, inp["d"], n)], axis=1)

    def run(self):
        """One pass over the sample; returns (elements per second, seconds)."""
        from oracle import s6_oracle as O
        inp = self.inp
        t0 = time.perf_counter()
        O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
               zoh=self.zoh, conv_w=inp["conv_w"], conv_b=inp["conv_b"], channels=self.ch, threads=self.cores)
        sec = time.perf_counter() - t0
        return len(self.ch) * inp["L"] / sec, sec

    def describe(self):
        L = self.inp["L"]
        n = len(self.ch)
        return (f"{n} seeded (b, channel) pairs x all {L} tokens of {WORKLOAD} ({n * L / 1e6:.1f}M elements; "
                f"float64 C loop, {self.cores} threads)")


def oracle_rate(inp, zoh, reps=3, threads=None):
    leg = OracleLeg(inp, zoh, threads)
    rates = [leg.run()[0] for _ in range(reps)]
    return statistics.median(rates) / 1e9, leg.cores, leg.describe()


# ------------------------------------------------------------------ rows
def time_events(fn, iters, stream):
    import torch
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(iters):
        fn()
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / iters


def row_decode(device, stream, pk, steps=96, pool=8):
    """Streaming decode: 256 sequences x 6 blocks x d1536 x N16 (147,456 state
    values per sequence), one token per step per block, fp32 state, in place."""
    import torch
    import selective_state_space_19_b200 as S
    Bt, d, N, K, blocks = 256, 1536, 16, 4, 6
    params = [{k: to_dev(v, device) for k, v in SI.decode_params(b).items()} for b in range(blocks)]
    h = [torch.zeros(Bt, d, N, device=device) for _ in range(blocks)]
    cs = [torch.zeros(Bt, d, K - 1, device=device) for _ in range(blocks)]
    toks = [[{k: to_dev(v, device) for k, v in SI.decode_tokens(s, b).items()} for b in range(blocks)]
            for s in range(pool)]
    ys = [torch.empty(Bt, d, device=device) for _ in range(blocks)]

    def one_cycle():
        for s in range(pool):
            for b in range(blocks):
                p, t = params[b], toks[s][b]
                S.s6_step(t["x"], t["dt"], t["B"], t["C"], p["A_log"], p["D"], p["conv_w"], h[b], cs[b], z_t=t["z"],
                          dt_bias=p["dt_bias"], conv_b=p["conv_b"], y_t=ys[b], stream=stream)

    with torch.cuda.stream(stream):
        one_cycle()  # warm-up outside capture
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            one_cycle()
        g.replay()
        torch.cuda.synchronize(device)
        reps = max(1, steps // pool)
        ms = time_events(g.replay, reps, stream)
    n_tok = pool * blocks  # launches per replay
    elems = n_tok * Bt * d
    per_launch_ms = ms / n_tok
    bytes_per = 2 * (N * 4) + 2 * (K - 1) * 4 + 4 * 4 + 2 * N * 4 / d  # h r+w, conv r+w, x/dt/z/y, B/C
    gbs = elems * bytes_per / (ms * 1e-3) / 1e9
    return {"workload": "decode: 256 seq x 6 blocks x d1536 x N16, K4, fp32, 1 token/step (CUDA graph of "
                        f"{n_tok} launches, {pool}-step input pool cycled)",
            "value": elems / (ms * 1e-3) / 1e9, "unit": "Gelem/s", "us_per_launch": per_launch_ms * 1e3,
            "us_per_token_all_blocks": per_launch_ms * 1e3 * blocks,
            "tokens_per_s_all_256_seqs": Bt / (per_launch_ms * 1e-3 * blocks),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "algorithmic_bytes_per_elem": bytes_per}}


def row_prefill(device, stream, pk, inp_dev, cfg, chunks=4, iters=10):
    """Chunked prefill of the long_seq workload: the sequence in `chunks` equal
    parts, each part a s6_conv_scan_fwd_from_state call started from the previous
    part's h_final and its last K-1 inputs (the first part from zeros)."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, d, N, K = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"], cfg["K"]
    zoh = int(bool(cfg["zoh"]))
    cuts = [L * i // chunks for i in range(chunks + 1)]
    t = inp_dev
    parts, hists = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        parts.append({k: t[k][:, lo:hi].contiguous() for k in ("x", "dt", "z", "B", "C")})
        hists.append(t["x"][:, hi - (K - 1):hi].transpose(1, 2).contiguous())
    ys = [torch.empty_like(p["x"]) for p in parts]
    hs = [torch.empty(Bt, d, N, device=device) for _ in parts]

    def prefill():
        for i, p in enumerate(parts):
            S.s6_conv_scan_fwd_from_state(p["x"], t["conv_w"], t["conv_b"], p["dt"], t["A_log"], p["B"], p["C"],
                                          t["D"], z=p["z"], dt_bias=t["dt_bias"], zoh_mode=zoh,
                                          h_init=hs[i - 1] if i else None, conv_hist=hists[i - 1] if i else None,
                                          y=ys[i], h_final=hs[i], stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            prefill()
        ms = time_events(prefill, iters, stream)
    assert S.s6_device_status(stream=stream, device=device) == 0
    elems = Bt * L * d
    ex2_per_s = elems * N / (ms * 1e-3)
    peak_ex2 = SMS * MUFU_PER_SM_CLK * pk["sm_max_mhz"] * 1e6
    return {"workload": f"chunked prefill: long_seq in {chunks} parts of {L // chunks} tokens, each started from "
                        "the previous part's (h, last K-1 inputs) by s6_conv_scan_fwd_from_state",
            "value": elems / (ms * 1e-3) / 1e9, "unit": "Gelem/s", "ms_per_prefill": ms, "launches": chunks,
            "roofline": {"bound": "alu", "achieved": ex2_per_s / 1e12, "peak": peak_ex2 / 1e12, "unit": "Tex2/s",
                         "frac": ex2_per_s / peak_ex2}}


def row_bwd(device, stream, pk, inp_dev, cfg, iters=3, fused=False):
    """Backward pass of the scan (s6_scan_bwd; with `fused`, of the conv + scan,
    s6_conv_scan_bwd) on the long_seq workload's inputs: the gradients of
    sum(dy * y) for a random dy."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, d, N = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"]
    t = inp_dev
    gen = torch.Generator(device=device).manual_seed(7)
    dy = torch.randn(Bt, L, d, device=device, generator=gen).to(t["x"].dtype)
    zoh = int(bool(cfg["zoh"]))

    def bwd():
        if fused:
            S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], dy,
                               z=t["z"], dt_bias=t["dt_bias"], zoh_mode=zoh, stream=stream)
        else:
            S.s6_scan_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], dy, z=t["z"], dt_bias=t["dt_bias"],
                          zoh_mode=zoh, stream=stream)

    with torch.cuda.stream(stream):
        bwd()
        torch.cuda.synchronize(device)
        ms = time_events(bwd, iters, stream)
    assert S.s6_device_status(stream=stream, device=device) == 0
    elems = Bt * L * d
    ex2_per_s = elems * N / (ms * 1e-3)
    peak_ex2 = SMS * MUFU_PER_SM_CLK * pk["sm_max_mhz"] * 1e6
    name = "s6_conv_scan_bwd (conv4 + SiLU + scan)" if fused else "s6_scan_bwd"
    write = "exact ZOH write" if zoh else "simplified write"
    return {"workload": f"{name} on long_seq (Bt16 L8192 d1536 N16, bf16 in, float32 gradients, gate, "
                        f"{write}): all gradients of sum(dy * y)",
            "value": elems / (ms * 1e-3) / 1e9, "unit": "Gelem/s", "ms_per_launch": ms,
            "roofline": {"bound": "alu", "achieved": ex2_per_s / 1e12, "peak": peak_ex2 / 1e12, "unit": "Tex2/s",
                         "frac": ex2_per_s / peak_ex2,
                         "note": "16 ex2 per element credited (the forward's); the kernel issues 48 "
                                 "(forward to checkpoints, chunk recompute, reverse)"}}


def row_train(device, stream, pk, inp_dev, cfg, iters=3):
    """A training step of the fused path on the long_seq inputs: the forward that
    also keeps the state before every 16th token (s6_conv_scan_fwd_ckpt), then the
    backward from those states (s6_conv_scan_bwd with ckpt), which runs no forward
    of its own.  Beside it, the same step with the backward that recomputes its
    checkpoints (s6_conv_scan_fwd, then s6_conv_scan_bwd)."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, d, N = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"]
    t = inp_dev
    gen = torch.Generator(device=device).manual_seed(7)
    dy = torch.randn(Bt, L, d, device=device, generator=gen).to(t["x"].dtype)
    zoh = int(bool(cfg["zoh"]))
    y = torch.empty_like(t["x"])
    h = torch.empty(Bt, d, N, device=device)
    ck = torch.empty(Bt, (L + S.CKPT_EVERY - 1) // S.CKPT_EVERY, d, N, device=device)
    args = (t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"])

    def fwd_ckpt():
        S.s6_conv_scan_fwd_ckpt(*args, z=t["z"], dt_bias=t["dt_bias"], zoh_mode=zoh, y=y, h_final=h, ckpt=ck,
                                stream=stream)

    def bwd_ckpt():
        S.s6_conv_scan_bwd(*args, dy, z=t["z"], dt_bias=t["dt_bias"], zoh_mode=zoh, ckpt=ck, stream=stream)

    def step():
        fwd_ckpt()
        bwd_ckpt()

    def step_recompute():
        S.s6_conv_scan_fwd(*args, z=t["z"], dt_bias=t["dt_bias"], zoh_mode=zoh, y=y, h_final=h, stream=stream)
        S.s6_conv_scan_bwd(*args, dy, z=t["z"], dt_bias=t["dt_bias"], zoh_mode=zoh, stream=stream)

    with torch.cuda.stream(stream):
        step()
        step_recompute()
        torch.cuda.synchronize(device)
        ms = time_events(step, iters, stream)
        ms_re = time_events(step_recompute, iters, stream)
        ms_f = time_events(fwd_ckpt, iters, stream)
        ms_b = time_events(bwd_ckpt, iters, stream)
    assert S.s6_device_status(stream=stream, device=device) == 0
    elems = Bt * L * d
    ex2_per_s = elems * 2 * N / (ms * 1e-3)
    peak_ex2 = SMS * MUFU_PER_SM_CLK * pk["sm_max_mhz"] * 1e6
    return {"workload": "training step of the fused path on long_seq (Bt16 L8192 d1536 N16, bf16 in, float32 "
                        "gradients, gate, simplified write): s6_conv_scan_fwd_ckpt (y, h_final and the state every "
                        "16 tokens), then s6_conv_scan_bwd from those states",
            "value": elems / (ms * 1e-3) / 1e9, "unit": "Gelem/s (forward + backward)", "ms_per_step": ms,
            "forward_ckpt_ms": ms_f, "backward_from_ckpt_ms": ms_b,
            "backward_from_ckpt_value": elems / (ms_b * 1e-3) / 1e9,
            "recomputing_step": {"ms_per_step": ms_re, "value": elems / (ms_re * 1e-3) / 1e9,
                                 "what": "s6_conv_scan_fwd, then s6_conv_scan_bwd running its own "
                                         "checkpointing forward"},
            "roofline": {"bound": "alu", "achieved": ex2_per_s / 1e12, "peak": peak_ex2 / 1e12, "unit": "Tex2/s",
                         "frac": ex2_per_s / peak_ex2,
                         "note": "16 ex2 per element credited to each of the forward and the backward; the "
                                 "kernels issue 48 (forward, chunk recompute, reverse)"}}


def row_scan(device, stream, pk, name, zoh=None, over=None, iters=20, label=None):
    """s6_conv_scan_fwd on another workload of the pages: per-launch CUDA-event
    times, median over `iters` launches, each after an L2 flush (cold) and, for
    inputs that fit in L2, also back to back (warm)."""
    import selective_state_space_19_b200 as S
    import torch
    over = dict(over or {})
    cfg = dict(SI.CONFIGS[name])
    cfg.update(over)
    zoh = bool(cfg["zoh"]) if zoh is None else bool(zoh)
    inp = SI.scan_inputs(name, **over)
    Bt, L, d, N = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"]
    t = {k: to_dev(inp[k], device) for k in ("x", "z", "B", "C", "dt", "A_log", "D", "dt_bias", "conv_w", "conv_b")}
    y = torch.empty_like(t["x"])
    h = torch.empty(Bt, d, N, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # 256 MB > L2

    def launch():
        S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"],
                           dt_bias=t["dt_bias"], zoh_mode=int(zoh), y=y, h_final=h, stream=stream)

    def timed_cold():
        ms = []
        with torch.cuda.stream(stream):
            for _ in range(3):
                launch()
            for _ in range(iters):
                flush.fill_(1)
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                s0.record(stream)
                launch()
                s1.record(stream)
                s1.synchronize()
                ms.append(s0.elapsed_time(s1))
        return statistics.median(ms)

    elems = Bt * L * d
    bpe = algorithmic_bytes_per_elem(cfg)
    in_bytes = elems * bpe
    ms_cold = timed_cold()
    assert S.s6_device_status(stream=stream, device=device) == 0
    peak_ex2 = SMS * MUFU_PER_SM_CLK * pk["sm_max_mhz"] * 1e6

    def roof(ms):
        ex2 = elems * N / (ms * 1e-3)
        gbs = in_bytes / (ms * 1e-3) / 1e9
        return {"bound": "alu", "achieved": ex2 / 1e12, "peak": peak_ex2 / 1e12, "unit": "Tex2/s",
                "frac": ex2 / peak_ex2,
                "hbm": {"achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                        "algorithmic_bytes_per_elem": bpe}}

    io = cfg["io"]
    desc = label or name
    row = {"workload": f"{desc}: Bt{Bt} L{L} d{d} N{N} K{cfg['K']}, {io} I/O, "
                       f"{'exact ZOH' if zoh else 'simplified'} write, fused conv4+SiLU + gate, h_final",
           "value": elems / (ms_cold * 1e-3) / 1e9, "unit": "Gelem/s", "ms_per_launch": ms_cold,
           "l2": "flushed before each launch (cold; the launch queued behind the flush)",
           "roofline": roof(ms_cold)}
    if in_bytes < 64e6:
        # back to back, between two events: the inputs stay in L2 and each
        # launch queues behind the previous one
        with torch.cuda.stream(stream):
            for _ in range(3):
                launch()
            ms_warm = time_events(launch, iters, stream)
        row["warm"] = {"value": elems / (ms_warm * 1e-3) / 1e9, "ms_per_launch": ms_warm,
                       "l2": "inputs resident in L2 (back-to-back launches, mean)", "roofline": roof(ms_warm)}
    return row


def row_random_A(device, stream, pk, inp_dev, cfg, iters=20):
    """The headline scan with A_log drawn at random (log U[0.5, 16] per (channel,
    state), so that no decay is a power of another) against the workload's
    A_log = log(n + 1), alternating launches of the two on the same inputs: the
    kernel must take the same time for both (16 live exponentials per element
    either way)."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, d, N = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"]
    t = inp_dev
    rng = np.random.default_rng(17)
    a_rand = torch.from_numpy(np.log(rng.uniform(0.5, 16.0, size=(d, N))).astype(np.float32)).to(device)
    y = torch.empty_like(t["x"])
    h = torch.empty(Bt, d, N, device=device)

    def launch(A_log):
        S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], A_log, t["B"], t["C"], t["D"], z=t["z"],
                           dt_bias=t["dt_bias"], zoh_mode=int(bool(cfg["zoh"])), y=y, h_final=h, stream=stream)

    ms = {"default": [], "random": []}
    with torch.cuda.stream(stream):
        for _ in range(3):
            launch(t["A_log"])
            launch(a_rand)
        for _ in range(iters):
            for key, A_log in (("default", t["A_log"]), ("random", a_rand)):
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                s0.record(stream)
                launch(A_log)
                s1.record(stream)
                s1.synchronize()
                ms[key].append(s0.elapsed_time(s1))
    assert S.s6_device_status(stream=stream, device=device) == 0
    elems = Bt * L * d
    md, mr = statistics.median(ms["default"]), statistics.median(ms["random"])
    peak_ex2 = SMS * MUFU_PER_SM_CLK * pk["sm_max_mhz"] * 1e6
    return {"workload": f"{WORKLOAD} scan with A_log ~ log U[0.5, 16] (alternating with the default A_log = "
                        f"log(n+1) on the same inputs)",
            "value": elems / (mr * 1e-3) / 1e9, "unit": "Gelem/s", "ms_per_launch": mr,
            "default_A_log_ms_per_launch": md, "time_ratio_random_over_default": mr / md,
            "roofline": {"bound": "alu", "achieved": elems * N / (mr * 1e-3) / 1e12, "peak": peak_ex2 / 1e12,
                         "unit": "Tex2/s", "frac": elems * N / (mr * 1e-3) / peak_ex2}}


def row_diag(device, stream, pk, inp_dev, cfg, iters=20):
    """The constant-decay cell (s6_diag_recurrence_fwd, decay 2^w per channel and
    state, write B*u, gate) on the long-sequence workload's u, z, B, C.  No
    exponential per token; per state three float32 operations (the write u*B,
    the update a*h + write, the readout h*C), so at N = 16 the FP32 FMA pipe
    binds before HBM (x, z read, y written, B / C rows)."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, d, N = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"]
    w = to_dev(SI.diag_log2_decay(d, N), device)
    t = inp_dev
    y = torch.empty_like(t["x"])
    h = torch.empty(Bt, d, N, device=device)

    def launch():
        S.s6_diag_recurrence_fwd(t["x"], t["B"], t["C"], t["D"], decay_source=S.S6_DECAY_CONST, log2_decay=w,
                                 z=t["z"], y=y, h_final=h, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            launch()
        ms = time_events(launch, iters, stream)
    assert S.s6_device_status(stream=stream, device=device) == 0
    elems = Bt * L * d
    s_ = 2 if cfg["io"] == "bf16" else 4
    bpe = 3 * s_ + 2 * N * s_ / d
    gbs = elems * bpe / (ms * 1e-3) / 1e9
    fma_per_elem = 3 * N
    fma_s = elems * fma_per_elem / (ms * 1e-3)
    fma_peak = SMS * 128 * pk["sm_max_mhz"] * 1e6  # FP32 FMA lanes x clock
    return {"workload": f"s6_diag_recurrence_fwd, constant decay, on {WORKLOAD}'s u, z, B, C (Bt{Bt} L{L} d{d} N{N}, "
                        f"{cfg['io']} I/O, gate, h_final)",
            "value": elems / (ms * 1e-3) / 1e9, "unit": "Gelem/s", "ms_per_launch": ms,
            "roofline": {"bound": "alu", "achieved": fma_s / 1e12, "peak": fma_peak / 1e12, "unit": "T FP32 op/s",
                         "frac": fma_s / fma_peak, "ops_per_elem": fma_per_elem,
                         "pipe": "FP32 FMA (148 SMs x 128 lanes x max SM clock)",
                         "hbm": {"achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                                 "algorithmic_bytes_per_elem": bpe, "peak_source": pk["source"]}}}


def row_block(device, stream, pk, Bt=256, blocks=6, reps=20):
    """Mamba-mini decode: one token for each of 256 sequences through all 6 blocks
    (s6_block_step: LayerNorm + int8 in_proj, conv + x_proj, dt_proj +
    recurrence, out_proj + residual), replayed as one CUDA graph per token."""
    import selective_state_space_19_b200 as S
    import torch
    cfgb = SI.MAMBA_MINI_BLOCK
    dm, di, N, R, K = (cfgb[k] for k in ("dm", "di", "N", "R", "K"))
    ws = [{k: to_dev(np.ascontiguousarray(v), device) for k, v in SI.block_weights(b).items()} for b in range(blocks)]
    cs = [torch.zeros(Bt, di, K - 1, device=device) for _ in range(blocks)]
    hs = [torch.zeros(Bt, di, N, device=device) for _ in range(blocks)]
    x = to_dev(SI.block_tokens(0, Bt=Bt), device)

    def token():
        for b in range(blocks):
            S.s6_block_step(x, cs[b], hs[b], ws[b], eps=cfgb["eps"], stream=stream)

    with torch.cuda.stream(stream):
        token()  # first call sizes the scratch, outside the capture
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            token()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(device)
        ms = time_events(g.replay, reps, stream)
    assert S.s6_device_status(stream=stream, device=device) == 0
    # per token step, all sequences and blocks
    state_bytes = blocks * Bt * di * (2 * N + 2 * (K - 1)) * 4
    weight_bytes = blocks * (2 * di * dm + (R + 2 * N) * di + di * R + dm * di)
    act_bytes = blocks * Bt * (2 * dm + 2 * 2 * di + 2 * di + 2 * (R + 2 * N)) * 4
    # in_proj and out_proj run on the tensor cores (TF32, two passes: the
    # activation's two terms); x_proj and dt_proj on the FP32 FMA pipe
    tc_flops = blocks * Bt * 2 * 2 * (2 * di * dm + dm * di)
    fma_flops = blocks * Bt * 2 * ((R + 2 * N) * di + di * R)
    total_bytes = state_bytes + weight_bytes + act_bytes
    gbs = total_bytes / (ms * 1e-3) / 1e9
    fp32_peak = SMS * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12
    tf32_peak = pk["bf16_tflops"] / 2  # dense TF32 is half the bf16 rate
    t_hbm = total_bytes / (pk["hbm_gbs"] * 1e9) * 1e3
    t_fma = fma_flops / (fp32_peak * 1e12) * 1e3
    t_tc = tc_flops / (tf32_peak * 1e12) * 1e3
    return {"workload": f"Mamba-mini decode: {Bt} sequences x {blocks} blocks (d_model {dm}, d_inner {di}, N {N}, "
                        f"dt rank {R}, conv {K}), int8 per-row weights, one token per sequence per step "
                        f"(CUDA graph of {blocks} s6_block_step calls)",
            "value": Bt / (ms * 1e-3), "unit": "tokens/s (all sequences)", "ms_per_token_step": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": t_hbm / ms, "bytes_per_step": total_bytes, "peak_source": pk["source"],
                         "note": "the state h read and written (302 MB of the 432 MB per token step) binds; "
                                 "the other bounds are far below it",
                         "tensor_tf32": {"flops_per_step": tc_flops, "peak_tflops": tf32_peak,
                                         "bound_ms": t_tc, "frac": t_tc / ms,
                                         "peak_note": "half the bf16 dense peak (" + pk["source"] + ")"},
                         "fp32_fma": {"flops_per_step": fma_flops, "peak_tflops": fp32_peak, "bound_ms": t_fma,
                                      "frac": t_fma / ms,
                                      "peak_note": "148 SMs x 128 FP32 lanes x 2 x max SM clock"}}}


def row_conv(device, stream, pk, inp_dev, cfg, iters=20):
    import selective_state_space_19_b200 as S
    import torch
    x, w, b = inp_dev["x"], inp_dev["conv_w"], inp_dev["conv_b"]
    out = torch.empty_like(x)
    with torch.cuda.stream(stream):
        for _ in range(3):
            S.causal_conv1d_silu_fwd(x, w, b, out=out, stream=stream)
        ms = time_events(lambda: S.causal_conv1d_silu_fwd(x, w, b, out=out, stream=stream), iters, stream)
    elems = cfg["Bt"] * cfg["L"] * cfg["d"]
    s = 2 if cfg["io"] == "bf16" else 4
    gbs = elems * 2 * s / (ms * 1e-3) / 1e9
    return {"workload": f"standalone conv4+SiLU on {WORKLOAD} x (Bt16 L8192 d1536 bf16)",
            "value": elems / (ms * 1e-3) / 1e9, "unit": "Gelem/s", "ms_per_launch": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "algorithmic_bytes_per_elem": 2 * s}}


# ------------------------------------------------------------------ main arms
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(v, world, device):
    """The slowest rank's time (the job is done when every rank is)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(elems_per_rank, world, total_ms_max, steps):
    """Whole-job Gelem/s: every rank scans its own batch (weak scaling), the time
    is the max over ranks of the timed region, divided into `steps` steps."""
    ms_per_step = total_ms_max / steps
    return world * elems_per_rank / (ms_per_step * 1e-3) / 1e9, ms_per_step


def rank_seed(base_seed, rank):
    """Each rank draws its own batch of the workload."""
    return base_seed + rank


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args):
    """The oracle arm: each step is one pass of the float64 oracle over the fixed
    sample of the CPU-baseline leg (not the whole workload); ms_per_step is the
    time of that pass."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = SI.CONFIGS[WORKLOAD]
    inp = SI.scan_inputs(WORKLOAD)
    leg = OracleLeg(inp, False)
    rates, secs = [], []
    for i in range(args.warmup + args.steps):
        r, sec = leg.run()
        if i >= args.warmup:
            rates.append(r)
            secs.append(sec)
    value = statistics.median(rates) / 1e9
    cores, desc = leg.cores, leg.describe()
    elems = cfg["Bt"] * cfg["L"] * cfg["d"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(secs) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy, long_seq recipe)",
            "config": {"workload": f"{WORKLOAD}: Bt16 L8192 d1536 N16 K4, bf16 inputs, simplified write, "
                                   "fused conv4+SiLU and SiLU(z) gate, h_final",
                       "global_batch": cfg["Bt"], "seq_len": cfg["L"], "parallelism": "oracle on host cores",
                       "l2": "n/a (host)", "step": f"one pass over the sample: {desc}"},
            "ms_per_step_full_workload_extrapolated": elems / (value * 1e9) * 1e3,
            "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import selective_state_space_19_b200 as S

    world, rank, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    S.lib()
    pk = peaks()
    cfg = dict(SI.CONFIGS[WORKLOAD])
    if args.case == "small":
        # profiling case: same kernel, distributions, batch and width, 1/4 of the
        # sequence (50M elements, ~300 MB of inputs: larger than L2; the
        # same 384 (sequence, channel-tile) chains as the full workload)
        cfg.update(L=2048)
        args.no_rows = args.no_e2e = args.no_cpu_baseline = True
    zoh = bool(cfg["zoh"])
    over = {k: cfg[k] for k in ("Bt", "L")}
    inp = SI.scan_inputs(WORKLOAD, seed=rank_seed(cfg["seed"], rank), **over)  # each rank its own batch
    Bt, L, d, N = cfg["Bt"], cfg["L"], cfg["d"], cfg["N"]
    elems = Bt * L * d
    stream = torch.cuda.Stream(device)
    keys = ("x", "z", "B", "C", "dt", "A_log", "D", "dt_bias", "conv_w", "conv_b")
    t = {k: to_dev(inp[k], device) for k in keys}
    y = torch.empty_like(t["x"])
    h = torch.empty(Bt, d, N, device=device)

    def step():
        S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"],
                           dt_bias=t["dt_bias"], zoh_mode=int(zoh), y=y, h_final=h, stream=stream)

    clocks = ClockSampler(local).start()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize(device)
        barrier(world)
        torch.cuda.synchronize(device)
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        host_t0 = time.time()
        t_all0.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize(device)
        host_t1 = time.time()
        barrier(world)
        torch.cuda.synchronize(device)
    clocks.stop()
    assert S.s6_device_status(stream=stream, device=device) == 0
    total_ms = t_all0.elapsed_time(t_all1)
    launch_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(total_ms, world, device)
    value, ms_per_step = job_throughput(elems, world, total_ms, args.steps)

    # roofline of the scan kernel: N exponentials per element on the MUFU pipe
    ex2_per_s = elems * N / (launch_ms * 1e-3)
    ck = clocks.summary(window=(host_t0, host_t1))
    peak_ex2 = SMS * MUFU_PER_SM_CLK * pk["sm_max_mhz"] * 1e6
    bpe = algorithmic_bytes_per_elem(cfg)
    gbs = elems * bpe / (launch_ms * 1e-3) / 1e9
    traffic, _ = recorded_traffic()
    roof = {"bound": "alu", "unit": "Tex2/s", "achieved": ex2_per_s / 1e12, "peak": peak_ex2 / 1e12,
            "frac": ex2_per_s / peak_ex2, "traffic": traffic,
            "pipe": "MUFU ex2 (148 SMs x 16/clk x max SM clock)",
            "peak_at_measured_clock": (SMS * MUFU_PER_SM_CLK * ck["sm_mhz"] * 1e6 / 1e12) if ck.get("sm_mhz") else None,
            "algorithmic_ex2_per_elem": N, "kernel": "s6_scan_kernel<bf16,16,2,64,2,conv,simplified>",
            "kernel_source_sha": kernel_source_sha(),
            "hbm": {"achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                    "algorithmic_bytes_per_elem": bpe, "peak_source": pk["source"]}}

    # ---- end to end: pinned host buffers -> device -> kernel -> host, every step
    e2e = None
    if not args.no_e2e:
        hin = {k: to_pinned(inp[k]) for k in ("x", "z", "B", "C", "dt")}
        hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        hh = torch.empty(h.shape, dtype=h.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in hin.values())
        d2h = hy.numel() * hy.element_size() + hh.numel() * hh.element_size()
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        # The batch moves in chunks of sequences on three streams -- host-to-
        # device copies, the scan, device-to-host copies -- so that the copies of
        # one chunk overlap the scan of another and the two directions overlap
        # each other.  Each chunk is one s6_conv_scan_fwd call on its sequences.
        nch = max(c for c in (1, 2, 4, 8, 16, 32) if c <= args.e2e_chunks and Bt % c == 0)
        cb = Bt // nch
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(nch)]
        ev_done = [torch.cuda.Event() for _ in range(nch)]  # scan of the chunk finished (inputs free)
        ev_out = [torch.cuda.Event() for _ in range(nch)]   # its outputs copied out (outputs free)
        for i in range(nch):
            ev_done[i].record(stream)
            ev_out[i].record(stream)

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            for i in range(nch):
                sl = slice(i * cb, (i + 1) * cb)
                s_in.wait_event(start)
                s_in.wait_event(ev_done[i])
                with torch.cuda.stream(s_in):
                    for k, v in hin.items():
                        t[k][sl].copy_(v[sl], non_blocking=True)
                ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                stream.wait_event(ev_out[i])
                S.s6_conv_scan_fwd(t["x"][sl], t["conv_w"], t["conv_b"], t["dt"][sl], t["A_log"], t["B"][sl],
                                   t["C"][sl], t["D"], z=t["z"][sl], dt_bias=t["dt_bias"], zoh_mode=int(zoh),
                                   y=y[sl], h_final=h[sl], stream=stream)
                ev_done[i].record(stream)
                s_out.wait_event(ev_done[i])
                with torch.cuda.stream(s_out):
                    hy[sl].copy_(y[sl], non_blocking=True)
                    hh[sl].copy_(h[sl], non_blocking=True)
                ev_out[i].record(s_out)
            for i in range(nch):
                stream.wait_event(ev_out[i])

        with torch.cuda.stream(stream):
            e2e_step()
            torch.cuda.synchronize(device)
            barrier(world)
            e_ms = time_events(e2e_step, e2e_steps, stream)
            barrier(world)
        # the chunked pipeline's result is the whole-batch scan's (within the
        # bf16 output rounding: chunks of few chains may take the associative split)
        with torch.cuda.stream(stream):
            step()
        torch.cuda.synchronize(device)
        ey = (hy.to(device).float() - y.float()).abs() / (1 + y.float().abs())
        eh = (hh.to(device) - h).abs() / (1 + h.abs())
        assert float(ey.max()) <= 1e-2 and float(eh.max()) <= 1e-4, (float(ey.max()), float(eh.max()))
        e_ms = max_over_ranks(e_ms, world, device)
        e2e = {"value": world * elems / (e_ms * 1e-3) / 1e9, "unit": "Gelem/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "steps": e2e_steps,
               "pipeline": f"{nch} chunks of {cb} sequences; copies in both directions overlap the scans"}

    rows = {}
    if not args.no_rows and rank == 0:
        rows["mamba_mini_simplified"] = row_scan(device, stream, pk, "mamba_mini", zoh=False)
        rows["mamba_mini_zoh"] = row_scan(device, stream, pk, "mamba_mini", zoh=True)
        rows["wide"] = row_scan(device, stream, pk, "wide")
        rows["single_prompt_assoc"] = row_scan(device, stream, pk, "long_seq", over=dict(Bt=1, L=65536),
                                               label="one long prompt, Bt1 L65536 (associative split)")
        rows["s6_step"] = row_decode(device, stream, pk)
        rows["s6_block_step"] = row_block(device, stream, pk)
        rows["long_seq_random_A_log"] = row_random_A(device, stream, pk, t, cfg)
        rows["s6_diag_recurrence_fwd_const"] = row_diag(device, stream, pk, t, cfg)
        rows["causal_conv1d_silu_fwd"] = row_conv(device, stream, pk, t, cfg)
        rows["s6_conv_scan_fwd_from_state"] = row_prefill(device, stream, pk, t, cfg)
        rows["s6_scan_bwd"] = row_bwd(device, stream, pk, t, cfg)
        rows["s6_conv_scan_bwd"] = row_bwd(device, stream, pk, t, cfg, fused=True)
        rows["s6_conv_scan_bwd_zoh"] = row_bwd(device, stream, pk, t, dict(cfg, zoh=True), fused=True)
        rows["train_step_conv_scan"] = row_train(device, stream, pk, t, cfg)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        g, cores, desc = oracle_rate(inp, zoh)
        cpu = {"value": g, "unit": "Gelem/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded numpy, long_seq recipe: x,z,B,C ~ N(0,1), dt_raw ~ 0.5 N(0,1), "
                        "dt_bias = softplus^-1(U[0.001,0.1]), A_log = log(n+1), D ~ U[0.5,1.5])",
                "config": {"workload": f"{WORKLOAD}: Bt16 L8192 d1536 N16 K4, bf16 I/O, fp32 state, simplified "
                                       "dt*B write, fused conv4+SiLU + SiLU(z) gate, h_final",
                           "global_batch": Bt * world, "seq_len": L, "d_inner": d, "d_state": N,
                           "io_dtype": "bf16", "state_dtype": "f32",
                           "parallelism": f"dp{world} (independent batches per GPU)",
                           "l2": "inputs larger than L2 (1.2 GB read per step), no flush"},
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
                "clocks": {"sm_mhz": ck.get("sm_mhz"), "sm_max_mhz": ck.get("sm_max_mhz"), "reasons": ck.get("reasons"),
                           "samples": ck.get("samples"), "sm_mhz_min": ck.get("sm_mhz_min"),
                           "power_w_max": ck.get("power_w_max"), "source": ck.get("source"),
                           "window": "timed region only"},
                "rows": rows}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_profile_case(case):
    """Small fixed cases for ncu captures of kernels outside the timed step:
    'bwd' -- three s6_scan_bwd calls on the long_seq recipe at Bt16 L1024 (the
    full workload's 384 chains, ~0.65 GB on the device); 'block' -- three decode
    token steps of 256 sequences through the 6 Mamba-mini blocks; 'mamba_mini'
    -- three fused scans of the Mamba-mini block workload (Bt8 L256 d1536,
    float32); 'diag' -- three constant-decay cells on the long_seq recipe at
    L = 2048 (50M elements; u, z, y 300 MB, larger than L2); 'train' -- three
    training steps of the fused path (s6_conv_scan_fwd_ckpt, then
    s6_conv_scan_bwd from its checkpoints) on the long_seq recipe at Bt16
    L1024."""
    import torch
    import selective_state_space_19_b200 as S
    dev = torch.device("cuda", 0)
    if case == "mamba_mini":
        inp = SI.scan_inputs("mamba_mini")
        t = {k: to_dev(inp[k], dev) for k in ("x", "z", "B", "C", "dt", "A_log", "D", "dt_bias", "conv_w", "conv_b")}
        for _ in range(3):
            S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                               z=t["z"], dt_bias=t["dt_bias"])
    elif case == "train":
        inp = SI.scan_inputs("long_seq", Bt=16, L=1024, seed=3)
        t = {k: to_dev(inp[k], dev) for k in ("x", "z", "B", "C", "dt", "A_log", "D", "dt_bias", "conv_w", "conv_b")}
        gen = torch.Generator(device=dev).manual_seed(7)
        dy = torch.randn(16, 1024, 1536, device=dev, generator=gen).to(torch.bfloat16)
        args = (t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"])
        for _ in range(3):
            _, _, ck = S.s6_conv_scan_fwd_ckpt(*args, z=t["z"], dt_bias=t["dt_bias"])
            S.s6_conv_scan_bwd(*args, dy, z=t["z"], dt_bias=t["dt_bias"], ckpt=ck)
    elif case == "diag":
        inp = SI.scan_inputs("long_seq", L=2048)
        t = {k: to_dev(inp[k], dev) for k in ("x", "z", "B", "C", "D")}
        w = to_dev(SI.diag_log2_decay(inp["x"].shape[2], 16), dev)
        for _ in range(3):
            S.s6_diag_recurrence_fwd(t["x"], t["B"], t["C"], t["D"], decay_source=S.S6_DECAY_CONST, log2_decay=w,
                                     z=t["z"])
    elif case == "bwd":
        inp = SI.scan_inputs("long_seq", Bt=16, L=1024, seed=3)
        t = {k: to_dev(inp[k], dev) for k in ("x", "z", "B", "C", "dt", "A_log", "D", "dt_bias")}
        gen = torch.Generator(device=dev).manual_seed(7)
        dy = torch.randn(16, 1024, 1536, device=dev, generator=gen).to(torch.bfloat16)
        for _ in range(3):
            S.s6_scan_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], dy, z=t["z"], dt_bias=t["dt_bias"])
    else:
        cfgb = SI.MAMBA_MINI_BLOCK
        ws = [{k: to_dev(np.ascontiguousarray(v), dev) for k, v in SI.block_weights(b).items()}
              for b in range(cfgb["blocks"])]
        cs = [torch.zeros(256, cfgb["di"], cfgb["K"] - 1, device=dev) for _ in ws]
        hs = [torch.zeros(256, cfgb["di"], cfgb["N"], device=dev) for _ in ws]
        x = to_dev(SI.block_tokens(0), dev)
        for _ in range(3):
            for b, w in enumerate(ws):
                S.s6_block_step(x, cs[b], hs[b], w, eps=cfgb["eps"])
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    print(f"profile case {case}: ok", flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", choices=["full", "small", "bwd", "block", "mamba_mini", "diag", "train"],
                    default="full",
                    help="small: the workload at L=2048 (for ncu captures); bwd, block, mamba_mini, diag, train: "
                         "small cases of the backward, the decode block, the Mamba-mini scan, the constant-decay "
                         "cell and a training step for captures (no JSON line)")
    ap.add_argument("--no-rows", action="store_true", help="skip the decode-step and standalone-conv rows")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="chunks of sequences in the end-to-end pipeline (the largest of 1, 2, 4, ... 32 that is at "
                         "most this and divides the batch)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.case in ("bwd", "block", "mamba_mini", "diag", "train"):
        return run_profile_case(args.case)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
