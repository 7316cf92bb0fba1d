#!/usr/bin/env python
"""Benchmark of the selective-SSM hot path on B200.

One step = one pass of the whole path on synthetic data:
  1. selective scan over the Mamba-2.8B-layer workload: batch 16, d_inner 5120,
     N 16, L 2048, bf16 u/delta/z/out, fp32 state, last_state returned;
  2. one generated token through 48 layers of selective_state_update at batch
     128, d_inner 4096, N 16, each layer's fp32 state (33.5 MB) updated in place
     (the 48 states, 1.6 GB, rotate so the state streams from HBM).

Reported: scan elements (B*D*L) per second, as the metric's value, with its
fraction of the MUFU roofline; the decode token-step in microseconds with its
fraction of HBM bandwidth.  Both inputs exceed L2 (126 MB), so no L2 flush is
needed between steps.  Timing uses CUDA events on the launching stream,
bracketed by a barrier and device synchronisation, max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own copy of the step on its own
inputs (weak scaling, no data-path collective); the value is the job total.
``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

METRIC = ("selective-scan Gelem/s (B·D·L) and % of roofline; "
          "decode-step µs at batch 128")
SCAN_WORKLOAD = "mamba_2p8b_layer"
SCAN_VARIANTS = ("euler", "zoh", "start_state", "bld")
PROFILES = ROOT / "profiles"
HBM_FALLBACK_GBS = 6650.0
HBM_NOMINAL_GBS = 8000.0
SM_MAX_MHZ_FALLBACK = 1965.0
BF16_TFLOPS_FALLBACK = 1590.0


# ----------------------------------------------------------------- helpers

def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", SM_MAX_MHZ_FALLBACK)),
                    "bf16_tflops": float(d.get("bf16_tflops", BF16_TFLOPS_FALLBACK)),
                    "source": "measured"}
        except Exception:  # noqa: BLE001
            pass
    return {"hbm_gbs": HBM_FALLBACK_GBS, "sm_max_mhz": SM_MAX_MHZ_FALLBACK,
            "bf16_tflops": BF16_TFLOPS_FALLBACK, "source": "fallback"}


def sources_digest() -> str:
    h = hashlib.sha256()
    csrc = ROOT / "selective_state_space_55_b200" / "csrc"
    for p in sorted(csrc.glob("*")) + [ROOT / "include" / "mamba_ssm.h"]:
        h.update(p.name.encode())
        h.update(p.read_bytes())
    return h.hexdigest()


def recorded_traffic(kernel: str, digest: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = PROFILES / "ncu_traffic.json"
    if not p.exists():
        return None
    try:
        rec = json.loads(p.read_text()).get(kernel)
    except Exception:  # noqa: BLE001
        return None
    if not rec or rec.get("sources_sha256") != digest:
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU through NVML (falls
    back to nvidia-smi) from a background thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, local_rank: int, period_s: float = 0.005):
        self.period = period_s
        self.samples: list[tuple[float, float, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = local_rank
            parts = [p for p in vis.split(",") if p.strip()]
            if parts and local_rank < len(parts) and parts[local_rank].strip().isdigit():
                idx = int(parts[local_rank])
            self._handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nvml = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # noqa: BLE001
            log(f"[bench] NVML unavailable ({e}); clocks via nvidia-smi")
        self.local_rank = local_rank

    def _poll(self):
        while not self._stop.is_set():
            t = time.time()
            try:
                if self._nvml is not None:
                    mhz = float(self._nvml.nvmlDeviceGetClockInfo(self._handle, self._nvml.NVML_CLOCK_SM))
                    reasons = int(self._nvml.nvmlDeviceGetCurrentClocksEventReasons(self._handle))
                else:
                    out = subprocess.run(
                        ["nvidia-smi", f"--id={self.local_rank}",
                         "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                         "--format=csv,noheader,nounits"],
                        capture_output=True, text=True, timeout=5).stdout.strip().split(",")
                    mhz, self.max_mhz = float(out[0]), float(out[1])
                    reasons = int(out[2].strip(), 16)
                self.samples.append((t, mhz, reasons))
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(self.period)

    def start(self):
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=10)

    def summary(self, t0: float, t1: float) -> dict:
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed_region"
        if not inside:
            inside, window = self.samples, "whole_run"
        reasons = set()
        for _, _, r in inside:
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    reasons.add(name)
        mhz = [s[1] for s in inside]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ----------------------------------------------------------------- workloads

class Workload:
    """Device-resident inputs and outputs of one step, and the calls that run it."""

    def __init__(self, rank: int, scan_batch: int | None = None, decode_layers: int | None = None,
                 only: str | None = None, scan_workload: str = SCAN_WORKLOAD,
                 scan_variant: str = "euler", scan_seqlen: int | None = None):
        from selective_state_space_55_b200 import inputs as I
        from selective_state_space_55_b200 import ops

        self.ops = ops
        self.only = only
        self.variant = scan_variant
        self.cfg = I.SCAN_CONFIGS[scan_workload]
        if scan_batch:
            self.cfg = self.cfg.resized(batch=scan_batch)
        if scan_seqlen:
            self.cfg = self.cfg.resized(seqlen=scan_seqlen)
        self.dcfg = I.DECODE_CONFIG
        if decode_layers:
            self.dcfg = I.DecodeConfig(self.dcfg.name, self.dcfg.batch, self.dcfg.dim,
                                       self.dcfg.dstate, decode_layers, self.dcfg.steps)
        c = self.cfg
        self.x = I.make_scan_inputs(c, "cuda", seed=rank_seed(rank))
        self.flags = 0
        if scan_variant == "bld":   # the same inputs in the (batch, seqlen, dim) layout
            for k in ("u", "delta", "z"):
                if self.x[k] is not None:
                    self.x[k] = self.x[k].transpose(1, 2).contiguous()
            self.flags = ops.MAMBA_FLAG_LAYOUT_BLD
        self.out = torch.empty_like(self.x["u"])
        self.last = torch.empty((c.batch, c.dim, c.dstate), dtype=torch.float32, device="cuda")
        self.h0 = None
        if scan_variant == "start_state":
            g = torch.Generator(device="cuda")
            g.manual_seed(rank_seed(rank) + 7)
            self.h0 = torch.randn((c.batch, c.dim, c.dstate), generator=g, device="cuda")
        ws = ops.scan_workspace_bytes(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype,
                                      flags=self.flags)
        self.ws = torch.empty(ws, dtype=torch.uint8, device="cuda") if ws else None
        self.plan = ops.scan_plan(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype, c.bc_dtype,
                                  sm_count=torch.cuda.get_device_properties(0).multi_processor_count,
                                  flags=self.flags)
        d = self.dcfg
        nl = 0 if only == "scan" else d.layers
        self.layers = [I.make_decode_layer(d, "cuda", seed=2000 + 100 * rank + i) for i in range(nl)]
        self.toks = [I.make_decode_token(d, "cuda", seed=3000 + 100 * rank + i) for i in range(nl)]
        self.douts = [torch.empty_like(t["x"]) for t in self.toks]
        self.graph = None

    def scan_kwargs(self) -> dict:
        return {"zoh": self.variant == "zoh", "initial_state": self.h0, "flags": self.flags}

    def scan(self):
        if self.only == "decode":
            return
        x = self.x
        self.ops.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                                    delta_bias=x["delta_bias"], softplus=True, out=self.out,
                                    last_state=self.last, workspace=self.ws, **self.scan_kwargs())

    def decode_layers(self):
        # Each layer updates its own state, so a layer's launch may overlap the
        # previous layer's (programmatic dependent launch, MAMBA_FLAG_PDL).
        for lay, tok, out in zip(self.layers, self.toks, self.douts):
            self.ops.selective_state_update(lay["state"], tok["x"], tok["dt"], lay["A"], tok["B"],
                                            tok["C"], D=lay["D"], z=tok["z"],
                                            dt_bias=lay["dt_bias"], out=out,
                                            flags=self.ops.MAMBA_FLAG_PDL)

    def capture_decode(self):
        """Capture the 48 state-update launches of one token in a CUDA graph."""
        if not self.layers:
            return
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.decode_layers()          # warm the launch path outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.decode_layers()
        torch.cuda.synchronize()

    def decode(self):
        if self.graph is not None:
            self.graph.replay()

    @property
    def launches_per_step(self) -> int:
        return (0 if self.only == "decode" else self.plan["launches"]) + len(self.layers)


def run_e2e(w: Workload, steps: int, warmup: int, rows: int = 0) -> dict:
    """Scan metric end to end through mamba_selective_scan_fwd_host: every step
    reads its inputs from pinned host memory and writes out / last_state back
    to pinned host memory; the library pipelines the copies by chunks of batch
    rows against the scans."""
    ops = w.ops
    x = w.x
    c = w.cfg
    names = ["u", "delta", "z", "B", "C", "A", "D", "delta_bias"]
    host = {k: (None if x[k] is None else x[k].cpu().pin_memory()) for k in names}
    h0_h = None if w.h0 is None else w.h0.cpu().pin_memory()
    out_h = torch.empty(w.out.shape, dtype=w.out.dtype, pin_memory=True)
    last_h = torch.empty(w.last.shape, dtype=w.last.dtype, pin_memory=True)
    zoh = w.variant == "zoh"
    flags = (ops.MAMBA_FLAG_ZOH if zoh else 0) | w.flags
    need = ops.scan_host_workspace_bytes(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype,
                                         c.bc_dtype, rows=rows, flags=flags)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    h2d += 0 if h0_h is None else h0_h.numel() * h0_h.element_size()
    d2h = out_h.numel() * out_h.element_size() + last_h.numel() * last_h.element_size()

    def step():
        ops.selective_scan_fwd_host(host["u"], host["delta"], host["A"], host["B"], host["C"],
                                    D=host["D"], z=host["z"], delta_bias=host["delta_bias"],
                                    softplus=True, out=out_h, last_state=last_h, rows=rows,
                                    workspace=ws, initial_state=h0_h, zoh=zoh, flags=w.flags)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e))
    chunk_rows = rows if rows > 0 else max(1, (c.batch + 7) // 8)
    pcie = pinned_copy_rates(host["u"], out_h)
    return {"ms_total": ms, "steps": steps, "h2d": h2d, "d2h": d2h, "rows": chunk_rows,
            "pcie": pcie}


def pinned_copy_rates(src_h: torch.Tensor, dst_h: torch.Tensor, reps: int = 5) -> dict:
    """Host-to-device and device-to-host copy rates (GB/s) of pinned host
    buffers, one cudaMemcpyAsync per copy on the current stream, timed with
    CUDA events: each direction alone, then both at once on two streams (the
    way the host-buffer scan overlaps them)."""
    dev_in = torch.empty(src_h.shape, dtype=src_h.dtype, device="cuda")
    dev_out = torch.empty(dst_h.shape, dtype=dst_h.dtype, device="cuda")
    nin = src_h.numel() * src_h.element_size()
    nout = dst_h.numel() * dst_h.element_size()

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e-3

    t_in = timed(lambda: dev_in.copy_(src_h, non_blocking=True))
    t_out = timed(lambda: dst_h.copy_(dev_out, non_blocking=True))
    side = torch.cuda.Stream()

    def both():
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            dst_h.copy_(dev_out, non_blocking=True)
        dev_in.copy_(src_h, non_blocking=True)
        torch.cuda.current_stream().wait_stream(side)

    t_both = timed(both)
    return {"h2d_gbs": round(nin / t_in / 1e9, 2), "d2h_gbs": round(nout / t_out / 1e9, 2),
            "both_directions_s": t_both, "h2d_bytes": nin, "d2h_bytes": nout,
            "h2d_gbs_while_d2h": round(nin / t_both / 1e9, 2)}


def _f64_block(x: dict, h0, b: int, d0: int, S: int, P: int) -> dict:
    """Float64 host copies of one sample block of a scan workload: batch row b,
    channels [d0, d0 + S), the first P time steps."""
    def cut(t):
        return None if t is None else t[b:b + 1, d0:d0 + S, :P].double().cpu().numpy().copy()
    return dict(u=cut(x["u"]), delta=cut(x["delta"]), z=cut(x["z"]),
                B=x["B"][b:b + 1, :, :P].double().cpu().numpy().copy(),
                C=x["C"][b:b + 1, :, :P].double().cpu().numpy().copy(),
                A=x["A"][d0:d0 + S].double().cpu().numpy().copy(),
                D=None if x["D"] is None else x["D"][d0:d0 + S].double().cpu().numpy().copy(),
                delta_bias=(None if x["delta_bias"] is None
                            else x["delta_bias"][d0:d0 + S].double().cpu().numpy().copy()),
                initial_state=None if h0 is None else h0[b:b + 1, d0:d0 + S].double().cpu().numpy().copy())


def _time_oracle_scan(ref, blocks: list, threads: int, target_s: float, zoh: bool):
    """Runs the oracle's scan over the sample blocks in turn (repeating them)
    with ``threads`` OpenMP threads until about ``target_s`` seconds; returns
    (elements, seconds, calls).  Inputs are float64 already, so only the
    oracle's own work is timed."""
    ref.set_num_threads(threads)
    done, t_total, calls = 0, 0.0, 0
    while True:
        for blk in blocks:
            t0 = time.perf_counter()
            ref.selective_scan(blk["u"], blk["delta"], blk["A"], blk["B"], blk["C"], D=blk["D"],
                               z=blk["z"], delta_bias=blk["delta_bias"], softplus=True, zoh=zoh,
                               initial_state=blk["initial_state"])
            t_total += time.perf_counter() - t0
            done += blk["u"].size
            calls += 1
            if t_total >= target_s:
                return done, t_total, calls


def cpu_baseline(w: Workload, target_s: float) -> dict:
    """The float64 oracle on the host cores over the same workload, on all
    cores and on one core, each for about ``target_s`` / 2 seconds.

    Sample blocks are (batch row, channel block, all L steps): two batch rows
    with all their channels for the layer shapes; for the million-token shape,
    two blocks of 32 channels (at least two per thread) over the whole
    sequence.  The one-core sample is one block of at most 2^21 elements.  The
    chains are independent, so elements per second over a sample are the rate
    over the whole workload."""
    from oracle import oracle
    ref = oracle.default()
    c = w.cfg
    zoh = w.variant == "zoh"
    all_threads = ref.num_threads()
    L = c.seqlen
    S_all = min(c.dim, max((1 << 25) // L, 2 * all_threads))
    S_one = max(1, min(c.dim, (1 << 21) // L))
    half = target_s / 2
    # two blocks: batch rows 0 and 1 (or two channel blocks of row 0)
    second = (1, 0) if c.batch > 1 else (0, S_all if 2 * S_all <= c.dim else 0)
    blocks_all = [_f64_block(w.x, w.h0, 0, 0, S_all, L),
                  _f64_block(w.x, w.h0, second[0], second[1], S_all, L)]
    blocks_one = [_f64_block(w.x, w.h0, 0, 0, S_one, L)]
    n_all, t_all, k_all = _time_oracle_scan(ref, blocks_all, all_threads, half, zoh)
    n_one, t_one, k_one = _time_oracle_scan(ref, blocks_one, 1, half, zoh)
    ref.set_num_threads(all_threads)
    v_all, v_one = n_all / t_all / 1e9, n_one / t_one / 1e9
    return {"value": v_all, "unit": "Gelem/s", "cores": all_threads, "kind": "oracle",
            "sample": f"{k_all} oracle calls over blocks of {c.name} (batch row x {S_all} "
                      f"channels x all L={L} steps; {n_all} elements) in {t_all:.1f} s on "
                      f"{all_threads} threads",
            "value_cores_all": v_all, "cores_all": all_threads,
            "value_cores_1": v_one, "cores_1": 1,
            "sample_cores_1": f"{k_one} oracle calls over {S_one} channels x L={L} of batch row 0 "
                              f"({n_one} elements) in {t_one:.1f} s on 1 thread",
            "host_cpu_count": os.cpu_count()}


def decode_cpu_baseline(w: Workload, target_s: float) -> dict | None:
    """The float64 update oracle on one token step of the decode workload:
    updates of one layer's state (batch 128 x 4096 x 16) repeated, on all
    cores and on one core (a 1/16 slice of the batch, scaled), each for about
    ``target_s`` / 2 seconds; reported per 48-layer token step."""
    if not w.layers:
        return None
    from oracle import oracle
    ref = oracle.default()
    d = w.dcfg
    lay, tok = w.layers[0], w.toks[0]
    f = lambda t: t.double().cpu().numpy().copy()  # noqa: E731
    args = dict(state=f(lay["state"]), x=f(tok["x"]), dt=f(tok["dt"]), A=f(lay["A"]), B=f(tok["B"]),
                C=f(tok["C"]), D=f(lay["D"]), z=f(tok["z"]), dt_bias=f(lay["dt_bias"]))
    rows1 = max(1, d.batch // 16)
    one = {k: (v[:rows1].copy() if k in ("state", "x", "dt", "B", "C", "z") else v)
           for k, v in args.items()}

    def timed(a, threads):
        ref.set_num_threads(threads)
        n, t_total = 0, 0.0
        while t_total < target_s / 2:
            t0 = time.perf_counter()
            ref.selective_state_update(a["state"], a["x"], a["dt"], a["A"], a["B"], a["C"],
                                       D=a["D"], z=a["z"], dt_bias=a["dt_bias"])
            t_total += time.perf_counter() - t0
            n += 1
        return t_total / n, n

    all_threads = ref.num_threads()
    t_all, n_all = timed(args, all_threads)
    t_one, n_one = timed(one, 1)
    ref.set_num_threads(all_threads)
    t_one_full = t_one * d.batch / rows1
    return {"kind": "oracle", "unit": "us per token step",
            "us_per_token_step_cores_all": round(t_all * d.layers * 1e6, 1), "cores_all": all_threads,
            "us_per_token_step_cores_1": round(t_one_full * d.layers * 1e6, 1), "cores_1": 1,
            "sample": f"{n_all} updates of one layer's state ({d.batch} x {d.dim} x {d.dstate}) "
                      f"on {all_threads} threads, {n_one} updates of {rows1} of its batch rows on "
                      f"1 thread (scaled by {d.batch // rows1}); a token step is {d.layers} layers"}


def bwd_cpu_baseline(cfg, x: dict, dout, target_s: float) -> dict:
    """The float64 oracle's backward pass on the host over whole batch rows of
    the workload, until about ``target_s`` seconds of CPU work."""
    from oracle import oracle
    ref = oracle.default()
    done, t_total, rows = 0, 0.0, 0
    for b in range(cfg.batch):
        sl = lambda t: None if t is None else t[b:b + 1].cpu()  # noqa: E731
        t0 = time.perf_counter()
        ref.selective_scan_bwd(sl(x["u"]), sl(x["delta"]), x["A"].cpu(), sl(x["B"]), sl(x["C"]),
                               sl(dout), D=x["D"].cpu(), z=sl(x["z"]),
                               delta_bias=x["delta_bias"].cpu())
        t_total += time.perf_counter() - t0
        done += cfg.dim * cfg.seqlen
        rows += 1
        if t_total >= target_s:
            break
    return {"value": done / t_total / 1e9, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} of {cfg.batch} batch rows of {cfg.name} backward ({cfg.dim} "
                      f"channels x L={cfg.seqlen}; {done} elements) in {t_total:.1f} s of oracle "
                      "time (the oracle's backward runs its chains in order)"}


def ssd_cpu_baseline(cfg, x: dict, target_s: float) -> dict:
    """The float64 oracle on the host cores over the Mamba-2 layer workload:
    batch rows in turn (all heads of a row per call), until about
    ``target_s`` seconds of CPU work or the whole batch."""
    from oracle import oracle
    ref = oracle.default()
    done, t_total, rows = 0, 0.0, 0
    for b in range(cfg.batch):
        sl = lambda t: None if t is None else t[b:b + 1].cpu()  # noqa: E731
        t0 = time.perf_counter()
        ref.ssd_scan(sl(x["x"]), sl(x["dt"]), x["A"].cpu(), sl(x["B"]), sl(x["C"]),
                     D=None if x["D"] is None else x["D"].cpu(), z=sl(x["z"]),
                     dt_bias=None if x["dt_bias"] is None else x["dt_bias"].cpu(),
                     initial_state=sl(x["initial_state"]))
        t_total += time.perf_counter() - t0
        done += cfg.seqlen * cfg.nheads * cfg.headdim
        rows += 1
        if t_total >= target_s:
            break
    return {"value": done / t_total / 1e9, "unit": "Gelem/s", "cores": ref.num_threads(),
            "kind": "oracle",
            "sample": f"{rows} of {cfg.batch} batch rows of {cfg.name} ({cfg.seqlen} tokens x "
                      f"{cfg.nheads} heads x {cfg.headdim}; {done} elements) in {t_total:.1f} s "
                      "of oracle time"}


# ----------------------------------------------------------------- distributed

_WORLD = 1
_REDUCE_DEVICE = "cuda"


def barrier():
    if _WORLD > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float) -> float:
    """Largest value of `v` over all ranks (each rank's device time)."""
    if _WORLD == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=_REDUCE_DEVICE)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of a rank's own synthetic inputs (every rank scans its own batch)."""
    return 1000 + rank


def job_gelem_per_s(world: int, elements_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's elements over the slowest rank's time."""
    return world * elements_per_rank * steps / (max_ms * 1e-3) / 1e9


# ----------------------------------------------------------------- arms

def bench_ours(args, rank, world, local):
    global _WORLD
    _WORLD = world
    from selective_state_space_55_b200 import build as cuda_build
    from selective_state_space_55_b200 import roofline as R

    if rank == 0:
        cuda_build.build()
    barrier()
    torch.cuda.set_device(local)
    partial = (args.only is not None or args.scan_batch or args.decode_layers or args.scan_seqlen
               or args.scan_workload != SCAN_WORKLOAD or args.scan_variant != "euler")
    w = Workload(rank, args.scan_batch, args.decode_layers, args.only, args.scan_workload,
                 args.scan_variant, args.scan_seqlen)
    c, d = w.cfg, w.dcfg
    w.capture_decode()
    for _ in range(args.warmup):
        w.scan()
        w.decode()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record()
    for e0, e1, e2 in ev:
        e0.record()
        w.scan()
        e1.record()
        w.decode()
        e2.record()
    end.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    sampler.stop()

    total_ms = max_over_ranks(start.elapsed_time(end))
    scan_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b, _ in ev))
    decode_ms = max_over_ranks(sum(b.elapsed_time(cc) for _, b, cc in ev))
    K = args.steps
    elems = c.elements
    value = job_gelem_per_s(world, elems, K, scan_ms)            # Gelem/s, whole job
    scan_launch_ms = scan_ms / K
    decode_step_us = decode_ms / K * 1e3

    peaks = measured_peaks()
    clocks = sampler.summary(t_wall0, t_wall1)
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    zoh = args.scan_variant == "zoh"
    # Peak on the method's own operation count (16 exponentials for Abar, 2
    # for softplus, 2 for the silu gate, and 1/Delta with the zero-order hold),
    # and on the count the bf16 kernel issues (its gate takes one tanh).
    mufu = R.scan_mufu_method(c.dstate, has_z=True, softplus=True, zoh=zoh)
    mufu_k = R.scan_mufu_per_element(c.dstate, has_z=True, softplus=True, zoh=zoh,
                                     io_bytes=c.io_dtype.itemsize)
    peak_elems = R.mufu_peak_elements_per_s(sms, peaks["sm_max_mhz"], mufu) / 1e9
    peak_kernel = R.mufu_peak_elements_per_s(sms, peaks["sm_max_mhz"], mufu_k) / 1e9
    achieved = elems / (scan_launch_ms * 1e-3) / 1e9               # per launch, this rank
    scan_bytes = R.scan_bytes(c.batch, c.dim, c.dstate, c.seqlen, 2, 2, True, True,
                              start_state=w.h0 is not None)
    upd_bytes = R.update_bytes(d.batch, d.dim, d.dstate, 2, 2, True)
    decode_gbs = upd_bytes * d.layers / (decode_ms / K * 1e-3) / 1e9
    digest = sources_digest()
    # Which kernel the plan runs, and its DRAM traffic where the record was
    # captured on this very workload (two lanes per channel on the 1.4B layer,
    # one lane on the 2.8B layer).
    scan_kernel = ("selective_scan_fwd_split_kernel" if w.plan.get("lanes_per_channel") == 2
                   else "selective_scan_fwd_kernel")
    recorded_on = {"selective_scan_fwd_kernel": ("mamba_2p8b_layer", 16),
                   "selective_scan_fwd_split_kernel": ("mamba_1p4b_layer", 8)}
    same_case = ((c.name, c.batch) == recorded_on[scan_kernel] and args.scan_variant == "euler"
                 and not args.scan_seqlen)
    scan_roof = {
        "bound": "alu", "pipe": f"MUFU (16 ops/clk/SM; {mufu} per element)",
        "kernel": scan_kernel,
        "achieved": round(achieved, 2), "peak": round(peak_elems, 2), "unit": "Gelem/s",
        "frac": round(achieved / peak_elems, 4),
        "peak_basis": f"{sms} SMs x 16 MUFU/clk x {peaks['sm_max_mhz']:.0f} MHz / {mufu} MUFU ops "
                      "per element in the method (16 exp for Abar, 2 softplus, 2 silu"
                      + (", 1 for 1/Delta" if zoh else "") + ")",
        "frac_at_measured_clock": (round(achieved / (peak_elems * clocks["sm_mhz"] / peaks["sm_max_mhz"]), 4)
                                   if clocks.get("sm_mhz") else None),
        "kernel_basis": {"mufu_per_element": mufu_k, "peak": round(peak_kernel, 2),
                         "frac": round(achieved / peak_kernel, 4),
                         "note": "the MUFU ops this kernel issues (bf16 inputs: the gate is one tanh)"},
        "algorithmic_bytes_per_launch": scan_bytes,
        "hbm_gbs": round(scan_bytes / (scan_launch_ms * 1e-3) / 1e9, 1),
        "traffic": recorded_traffic(scan_kernel, digest) if same_case else None,
    }
    state_bytes = 2 * d.batch * d.dim * d.dstate * 4
    state_gbs = state_bytes * d.layers / (decode_ms / K * 1e-3) / 1e9
    decode_roof = {"bound": "hbm", "kernel": "state_update_bulk_kernel",
                   "achieved": round(decode_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "frac": round(decode_gbs / peaks["hbm_gbs"], 4),
                   "peak_source": peaks["source"],
                   "frac_of_nominal": round(decode_gbs / HBM_NOMINAL_GBS, 4),
                   "nominal_peak": HBM_NOMINAL_GBS,
                   "state_traffic": {"bytes_per_layer": state_bytes, "achieved": round(state_gbs, 1),
                                     "frac_of_measured": round(state_gbs / peaks["hbm_gbs"], 4),
                                     "frac_of_nominal": round(state_gbs / HBM_NOMINAL_GBS, 4),
                                     "target": "state traffic at >= 75% of HBM peak; reported against "
                                               "both the measured copy peak and the nominal 8 TB/s"},
                   "algorithmic_bytes_per_launch": upd_bytes,
                   "traffic": recorded_traffic("state_update_bulk_kernel", digest)}
    decode = {
        "workload": f"decode_b128: {d.layers} layers x state ({d.batch}, {d.dim}, {d.dstate}) fp32, "
                    "bf16 x/dt/z/B/C/out, one CUDA graph per token, each layer's launch a "
                    "programmatic dependent launch (MAMBA_FLAG_PDL: distinct states per layer)",
        "us_per_token_step": round(decode_step_us, 2),
        "us_per_layer": round(decode_step_us / d.layers, 3),
        "roofline": decode_roof,
        "tokens_per_s": round(world * d.batch / (decode_step_us * 1e-6), 1),
    }
    # The step's dominant kernel (largest share of the step time) gets the
    # top-level roofline; the other kernel's stays in its own object.
    scan_share = scan_ms / max(scan_ms + decode_ms, 1e-9)
    scan_roof["share_of_step"] = round(scan_share, 4)
    decode_roof["share_of_step"] = round(1 - scan_share, 4)
    roof = scan_roof if scan_ms >= decode_ms else decode_roof

    e2e = None
    if not args.no_e2e and args.only != "decode":
        r = run_e2e(w, max(1, min(K, args.e2e_steps)), 2, args.e2e_rows)
        e2e_value = job_gelem_per_s(world, elems, r["steps"], r["ms_total"])
        pc = r["pcie"]
        # Both directions run at once in the host-buffer pipeline, so the copy
        # bound of a step is the slower direction at the rates measured alone.
        copy_s = max(r["h2d"] / (pc["h2d_gbs"] * 1e9), r["d2h"] / (pc["d2h_gbs"] * 1e9))
        pcie_bound = world * elems / copy_s / 1e9
        e2e = {"value": round(e2e_value, 3),
               "unit": "Gelem/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
               "steps": r["steps"],
               "pcie": {"h2d_gbs": pc["h2d_gbs"], "d2h_gbs": pc["d2h_gbs"],
                        "h2d_gbs_while_d2h": pc["h2d_gbs_while_d2h"],
                        "copy_bound_gelem_s": round(pcie_bound, 3),
                        "frac_of_copy_bound": round(e2e_value / pcie_bound, 4),
                        "method": "pinned cudaMemcpyAsync of the u tensor (h2d) and the out "
                                  "tensor (d2h), CUDA events, same run"},
               "path": "mamba_selective_scan_fwd_host: pinned host u/delta/z/B/C/A/D/bias -> "
                       f"device in chunks of {r['rows']} batch rows, scans overlapped with the "
                       "copies in and out -> out/last_state in pinned host memory"}

    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and args.only != "decode"
            and w.variant != "bld"):   # the oracle's blocks read (batch, dim, seqlen) rows
        cpu = cpu_baseline(w, args.cpu_seconds)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only != "scan":
        decode["cpu_baseline"] = decode_cpu_baseline(w, args.cpu_seconds / 2)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "Gelem/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; shapes and distributions of the pages' workloads)",
            "config": {
                "workload": f"{c.name} scan ({c.batch}x{c.dim}, N={c.dstate}, L={c.seqlen}, "
                            "bf16 in/out, fp32 state, last_state"
                            + ("" if w.variant == "euler" else f"; variant {w.variant}")
                            + ") + decode_b128 token step "
                            f"({d.layers} layers, batch {d.batch}, d_inner {d.dim}, N {d.dstate})",
                "io_dtype": "bf16", "state_dtype": "f32", "global_batch": world * c.batch,
                "seq_len": c.seqlen, "parallelism": f"replicas{world}" if world > 1 else "single",
                "l2": "inputs larger than L2 (1.0 GB scan inputs, 1.6 GB rotating decode state)",
                "scan_plan": w.plan,
            },
            "scan_ms_per_step": round(scan_ms / K, 4),
            "roofline": roof,
            "scan_roofline": scan_roof,
            "decode": decode,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": K * w.launches_per_step,
            "clocks": clocks,
            "sources_sha256": digest[:16],
        }
        if partial:
            line["partial_case"] = {"only": args.only, "scan_batch": args.scan_batch,
                                    "scan_seqlen": args.scan_seqlen,
                                    "decode_layers": args.decode_layers,
                                    "scan_workload": args.scan_workload,
                                    "scan_variant": args.scan_variant,
                                    "note": "profiling case, not the benchmark workload"}
        print(json.dumps(line), flush=True)


def bench_conv(args, rank, world, local):
    """Measurement case: the block's short causal convolution (W = 4, bf16) on the
    Mamba-2.8B layer shape (prefill) and 48 decode layers of batch 128 x 4096
    (one CUDA graph per token), each against the HBM roofline."""
    global _WORLD
    _WORLD = world
    from selective_state_space_55_b200 import build as cuda_build
    from selective_state_space_55_b200 import inputs as I
    from selective_state_space_55_b200 import ops

    if rank == 0:
        cuda_build.build()
    barrier()
    torch.cuda.set_device(local)
    c, d, W, bf = I.SCAN_CONFIGS[SCAN_WORKLOAD], I.DECODE_CONFIG, 4, torch.bfloat16
    g = torch.Generator(device="cuda")
    g.manual_seed(rank_seed(rank) + 11)
    x = torch.randn(c.batch, c.dim, c.seqlen, generator=g, device="cuda").to(bf)
    w = torch.randn(c.dim, W, generator=g, device="cuda") / W
    bias = torch.randn(c.dim, generator=g, device="cuda")
    out = torch.empty_like(x)
    fin = torch.empty(c.batch, c.dim, W, dtype=bf, device="cuda")
    lay = [dict(st=torch.randn(d.batch, d.dim, W, generator=g, device="cuda").to(bf),
                x=torch.randn(d.batch, d.dim, generator=g, device="cuda").to(bf),
                w=torch.randn(d.dim, W, generator=g, device="cuda") / W,
                b=torch.randn(d.dim, generator=g, device="cuda"),
                out=torch.empty(d.batch, d.dim, dtype=bf, device="cuda")) for _ in range(d.layers)]

    def prefill():
        ops.causal_conv1d_fwd(x, w, bias=bias, out=out, final_conv_state=fin)

    def decode():
        # each layer has its own conv state: dependent launches (MAMBA_FLAG_PDL)
        for ly in lay:
            ops.causal_conv1d_update(ly["st"], ly["x"], ly["w"], bias=ly["b"], out=ly["out"],
                                     flags=ops.MAMBA_FLAG_PDL)

    decode()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        decode()
    for _ in range(args.warmup):
        prefill()
        graph.replay()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for e0, e1, e2 in ev:
        e0.record()
        prefill()
        e1.record()
        graph.replay()
        e2.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    sampler.stop()
    pre_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b, _ in ev)) / K
    dec_ms = max_over_ranks(sum(b.elapsed_time(e) for _, b, e in ev)) / K
    chains_p, chains_d = c.batch * c.dim, d.batch * d.dim
    pre_bytes = c.elements * 2 * 2 + chains_p * W * 2 + c.dim * (W + 1) * 4
    dec_bytes = chains_d * (2 * W * 2 + 2 * 2) + d.dim * (W + 1) * 4        # per layer
    peaks = measured_peaks()
    pre_gbs = pre_bytes / (pre_ms * 1e-3) / 1e9
    dec_gbs = dec_bytes * d.layers / (dec_ms * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": "causal conv1d GB/s (prefill, Mamba-2.8B layer shape)", "value": round(world * pre_gbs, 1),
            "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(pre_ms + dec_ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)",
            "config": {"workload": f"causal conv1d W={W} bf16: prefill ({c.batch}x{c.dim}x{c.seqlen}) "
                                   f"+ decode update ({d.layers} layers x {d.batch}x{d.dim}, CUDA graph)"},
            "prefill": {"ms": round(pre_ms, 4), "bytes": pre_bytes,
                        "roofline": {"bound": "hbm", "achieved": round(pre_gbs, 1), "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "frac": round(pre_gbs / peaks["hbm_gbs"], 4)}},
            "decode": {"us_per_layer": round(dec_ms * 1e3 / d.layers, 3), "bytes_per_layer": dec_bytes,
                       "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": peaks["hbm_gbs"],
                                    "unit": "GB/s", "frac": round(dec_gbs / peaks["hbm_gbs"], 4)}},
            "gpu_launches": K * (1 + 1 + d.layers),
            "clocks": sampler.summary(t0, t1),
            "partial_case": {"only": "conv", "note": "measurement of the short convolution, not the benchmark workload"},
        }
        print(json.dumps(line), flush=True)


def bench_bwd(args, rank, world, local):
    """Measurement case: the backward pass of the scan (checkpoint pass + adjoint)
    on the Mamba-2.8B layer shape, gate, D and bias on, dout random; with
    ``--scan-variant bld`` the activations and their gradients are
    (batch, seqlen, dim), with ``--scan-variant zoh`` the input term is the
    zero-order hold's."""
    if args.scan_variant not in ("euler", "bld", "zoh"):
        raise SystemExit("--only bwd takes --scan-variant euler, bld or zoh")
    bld = args.scan_variant == "bld"
    zoh = args.scan_variant == "zoh"
    global _WORLD
    _WORLD = world
    from selective_state_space_55_b200 import build as cuda_build
    from selective_state_space_55_b200 import inputs as I
    from selective_state_space_55_b200 import ops
    from selective_state_space_55_b200 import roofline as R

    if rank == 0:
        cuda_build.build()
    barrier()
    torch.cuda.set_device(local)
    c = I.SCAN_CONFIGS[SCAN_WORKLOAD]
    if args.scan_batch:
        c = c.resized(batch=args.scan_batch)
    x = I.make_scan_inputs(c, "cuda", seed=rank_seed(rank))
    g = torch.Generator(device="cuda")
    g.manual_seed(rank_seed(rank) + 13)
    dout = torch.randn(c.batch, c.dim, c.seqlen, generator=g, device="cuda").to(c.io_dtype)
    ws = torch.empty(ops.scan_bwd_workspace_bytes(c.batch, c.dim, c.dstate, c.seqlen, c.io_dtype,
                                                  c.bc_dtype), dtype=torch.uint8, device="cuda")
    act = {k: x[k] for k in ("u", "delta", "z")}
    if bld:   # the same values in the (batch, seqlen, dim) layout
        act = {k: (None if v is None else v.transpose(1, 2).contiguous()) for k, v in act.items()}
        dout = dout.transpose(1, 2).contiguous()

    def step():
        return ops.selective_scan_bwd(act["u"], act["delta"], x["A"], x["B"], x["C"], dout, D=x["D"],
                                      z=act["z"], delta_bias=x["delta_bias"], workspace=ws,
                                      layout="bld" if bld else "bdl", zoh=zoh)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(K):
        step()
    e.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    sampler.stop()
    ms = max_over_ranks(s.elapsed_time(e)) / K
    peaks = measured_peaks()
    # MUFU ops per element over both launches.  Checkpoint pass: 16 ex2 + the
    # softplus (2).  Adjoint: 16 ex2 for the block's Abar (formed once while the
    # states are recomputed and kept for the way back), the softplus again (2),
    # its derivative sigmoid (2) and the gate's sigmoid (2).
    mufu = (16 + 2) + (16 + 2 + 2 + 2)
    if zoh:   # the gain's 1 / Delta, once per step in each launch
        mufu += 2
    # An adjoint that forms Abar a second time on the way back issues 16 more;
    # the fraction on that basis is reported beside this one.
    mufu_twice = mufu + 16
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    peak = R.mufu_peak_elements_per_s(sms, peaks["sm_max_mhz"], mufu) / 1e9
    peak_twice = R.mufu_peak_elements_per_s(sms, peaks["sm_max_mhz"], mufu_twice) / 1e9
    value = world * c.elements / (ms * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": "selective-scan backward Gelem/s (Mamba-2.8B layer shape)", "value": round(value, 3),
            "unit": "Gelem/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)",
            "config": {"workload": f"{c.name} backward ({c.batch}x{c.dim}, N={c.dstate}, L={c.seqlen}, "
                                   "bf16, gate/D/bias, checkpoint pass + adjoint)",
                       "input_term": "zero-order hold" if zoh else "Euler",
                       "activations": "(batch, seqlen, dim)" if bld else "(batch, dim, seqlen)",
                       "checkpoint_bytes": ws.numel()},
            "roofline": {"bound": "alu", "pipe": f"MUFU ({mufu} per element, both launches)",
                         "kernel": "selective_scan_bwd_kernel",
                         "achieved": round(value / world, 2), "peak": round(peak, 2), "unit": "Gelem/s",
                         "frac": round(value / world / peak, 4),
                         f"peak_{mufu_twice}_op_basis": round(peak_twice, 2),
                         f"frac_{mufu_twice}_op_basis": round(value / world / peak_twice, 4),
                         "traffic": (recorded_traffic("selective_scan_bwd_kernel", sources_digest())
                                     if c.batch == 16 and not bld and not zoh else None)},
            "gpu_launches": K * 2,
            "clocks": sampler.summary(t0, t1),
            "cpu_baseline": (None if args.no_cpu_baseline or bld or zoh
                             else bwd_cpu_baseline(c, x, dout, args.cpu_seconds)),
            "partial_case": {"only": "bwd", "scan_batch": args.scan_batch, "scan_variant": args.scan_variant,
                             "note": "measurement of the backward pass, not the benchmark workload"},
        }
        print(json.dumps(line), flush=True)


def bench_ssd(args, rank, world, local):
    """Measurement case: the Mamba-2 layer (scalar A per head) on the tensor
    cores, Mamba-2 2.7B layer shape (batch 16, L 2048, 80 heads x 64, state
    128, one group), gate, D and bias on, final state returned."""
    global _WORLD
    _WORLD = world
    from selective_state_space_55_b200 import build as cuda_build
    from selective_state_space_55_b200 import inputs as I
    from selective_state_space_55_b200 import ops
    from selective_state_space_55_b200 import roofline as R

    if rank == 0:
        cuda_build.build()
    barrier()
    torch.cuda.set_device(local)
    c = I.SSD_CONFIGS["mamba2_2p7b_layer"]
    if args.scan_batch:
        c = c.resized(batch=args.scan_batch)
    x = I.make_ssd_inputs(c, "cuda", seed=rank_seed(rank))
    out = torch.empty_like(x["x"])
    final = torch.empty(c.batch, c.nheads, c.headdim, c.dstate, dtype=torch.float32, device="cuda")

    def step():
        ops.ssd_chunk_scan_fwd(x["x"], x["dt"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                               dt_bias=x["dt_bias"], out=out, final_state=final)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(K):
        step()
    e.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    sampler.stop()
    ms = max_over_ranks(s.elapsed_time(e)) / K
    peaks = measured_peaks()
    nbytes = R.ssd_bytes(c.batch, c.seqlen, c.nheads, c.headdim, c.ngroups, c.dstate, c.has_z)
    flops = R.ssd_chunk_flops(c.batch, c.seqlen, c.nheads, c.headdim, c.dstate)
    issued = R.ssd_issued_flops(c.batch, c.seqlen, c.nheads, c.headdim, c.dstate)
    gbs = nbytes / (ms * 1e-3) / 1e9
    tfs = issued / (ms * 1e-3) / 1e12
    traffic = recorded_traffic("ssd_chunk_scan_kernel", sources_digest())
    value = world * c.elements / (ms * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": "Mamba-2 layer Gelem/s (B·L·heads·headdim)", "value": round(value, 3),
            "unit": "Gelem/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
            "config": {"workload": f"{c.name} ({c.batch}x{c.seqlen}, {c.nheads} heads x {c.headdim}, "
                                   f"N={c.dstate}, groups={c.ngroups}, chunk 128, bf16, gate/D/bias, "
                                   "final state)",
                       "inputs_exceed_l2": nbytes > 126e6},
            "roofline": {"bound": "hbm", "kernel": "ssd_chunk_scan_kernel", "achieved": round(gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "traffic": traffic if c.batch == 16 else None,
                         "bytes_per_step": nbytes},
            "tensor": {"issued_tflops": round(tfs, 1), "peak": peaks["bf16_tflops"],
                       "frac": round(tfs / peaks["bf16_tflops"], 4), "issued_flops_per_step": issued,
                       "algorithmic_flops_per_step": flops,
                       "algorithmic_tflops": round(flops / (ms * 1e-3) / 1e12, 1)},
            "gpu_launches": K,
            "clocks": sampler.summary(t0, t1),
            "cpu_baseline": (None if args.no_cpu_baseline
                             else ssd_cpu_baseline(c, x, args.cpu_seconds)),
            "partial_case": {"only": "ssd", "scan_batch": args.scan_batch,
                             "note": "measurement of the Mamba-2 layer, not the benchmark workload"},
        }
        print(json.dumps(line), flush=True)


def bench_reference(args, rank, world):
    """The float64 CPU oracle, on the same workload's metric, a bounded sample
    per step (rank 0 only)."""
    if rank != 0:
        return
    import numpy as np  # noqa: F401
    from oracle import oracle
    from selective_state_space_55_b200 import inputs as I

    ref = oracle.default()
    cfg = I.SCAN_CONFIGS[SCAN_WORKLOAD]
    L = cfg.seqlen
    small = cfg.resized(batch=1, dim=min(cfg.dim, 4096))
    x = I.make_scan_inputs(small, "cpu", seed=1000)

    def run(S):
        sl = lambda t: None if t is None else t[0:1, :S]  # noqa: E731
        t0 = time.perf_counter()
        ref.selective_scan(sl(x["u"]), sl(x["delta"]), x["A"][:S], x["B"][0:1], x["C"][0:1],
                           D=x["D"][:S], z=sl(x["z"]), delta_bias=x["delta_bias"][:S], softplus=True)
        return time.perf_counter() - t0

    budget_s = args.reference_seconds
    t1 = run(8) / 8
    per_step = budget_s / max(1, args.steps + args.warmup)
    S = int(max(1, min(small.dim, per_step / max(t1, 1e-9))))
    for _ in range(args.warmup):
        run(S)
    times = [run(S) for _ in range(args.steps)]
    total = sum(times)
    value = S * L * args.steps / total / 1e9
    sample = (f"{S} chains (batch row 0, channels 0..{S - 1}) x L={L} of {SCAN_WORKLOAD} per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Gelem/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{SCAN_WORKLOAD} scan, sampled chains (float64 CPU oracle)",
                   "seq_len": L},
        "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": ref.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-rows", type=int, default=0,
                    help="batch rows per chunk of the host-buffer call (0: automatic)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="budget of the whole --impl reference run")
    ap.add_argument("--only", choices=["scan", "decode", "conv", "bwd", "ssd"], default=None,
                    help="profiling case: one half of the step; conv: the short convolution; "
                         "bwd: the backward pass; ssd: the Mamba-2 layer")
    ap.add_argument("--scan-batch", type=int, default=None,
                    help="profiling case: smaller scan batch")
    ap.add_argument("--scan-seqlen", type=int, default=None,
                    help="profiling case: shorter scan sequence")
    ap.add_argument("--decode-layers", type=int, default=None,
                    help="profiling case: fewer decode layers")
    ap.add_argument("--scan-workload", default=SCAN_WORKLOAD,
                    choices=["mamba_1p4b_layer", "mamba_2p8b_layer", "long_dna_1m"],
                    help="measurement case: another scan workload")
    ap.add_argument("--scan-variant", default="euler", choices=SCAN_VARIANTS,
                    help="measurement case: zero-order-hold input term, or a start state")
    args = ap.parse_args()
    if args.warmup < 3:
        log("[bench] warm-up raised to 3 steps (minimum)")
        args.warmup = 3

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        log(f"[bench] note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")

    if args.impl == "reference":
        bench_reference(args, rank, world)
        return

    if world > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300),
            device_id=torch.device("cuda", local))
    try:
        if args.only == "conv":
            bench_conv(args, rank, world, local)
        elif args.only == "bwd":
            bench_bwd(args, rank, world, local)
        elif args.only == "ssd":
            bench_ssd(args, rank, world, local)
        else:
            bench_ours(args, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
