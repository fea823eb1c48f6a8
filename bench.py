#!/usr/bin/env python3
"""Bench of the quantized gated delta-rule decode step (libsq on B200).

One step = one call of the whole hot path (sq_decode_step: unpack, gated delta update, output,
dual-axis refit, requantize and repack in place) over one batch of synthetic requests. The
default workload is the serving pool, the largest single-GPU workload: a pool of 1024 slots,
512 active requests chosen by a seeded permutation, 32 heads, d_k = d_v = 128, per-head widths
{2, 4, 6} (mean 4) plus 2 fp16 pivot heads, bf16 q/k/v, updated in place.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload pool|gdn|kda|window|chunk|split] [--impl ours|reference]

The K timed steps run as RUNS separate timed regions (each K steps, bracketed by a barrier and a
device synchronization, device-timed with CUDA events, the max over ranks); the reported time
is the median region. L2 is flushed before every timed step.

The chunk workload is the GDN layer advanced 8 tokens per call (sq_decode_chunk); one step is
one call, and it counts batch x 8 request-steps. The split workload is the GDN layer through
sq_decode_step_split (update on one stream, refit + requantize on a second); a step ends when
both streams are done.

Prints one JSON line (rank 0). Multi-GPU: launched by torchrun, one process per GPU, each rank
decoding its own requests (weak scaling, no collective on the data path); times are device
times (CUDA events) and the max over ranks is reported. The reference arm (--impl reference)
times the CPU oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_recurrent_state_gated_b200 import dist  # noqa: E402
from bit_recurrent_state_gated_b200 import workloads as W  # noqa: E402

METRIC = "quantized delta-rule decode: request-steps/s and state HBM GB/s vs peak"
UNIT = "request-steps/s"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB of L2
L2_BYTES = 126 << 20
E2E_SETS = 8


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="pool", choices=["tiny", "gdn", "kda", "pool", "window",
                                                          "chunk", "split"])
    ap.add_argument("--runs", type=int, default=5, help="timed regions of K steps (median)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cold-window", action="store_true",
                    help="windowed workloads: run one whole window after the cold quantize, "
                         "untimed, and exit (a fixed launch sequence for the profiler)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the measured copy bandwidth is the peak used)

# ---- byte accounting ---------------------------------------------------------------------------

def algorithmic_bytes(wl: W.Workload, slot_bytes: int) -> dict:
    """Bytes one request-step must move (`total`): the packed state (codes, scales, fp16 units)
    read and written, q/k/v read, alpha/beta read, o written, the slot index read. Windowed
    layouts read the frozen block every token and write it once per window; the low-rank side
    state they keep for the open window (a header with the cumulative gate, one term per token:
    the token's k in the I/O type and b / g in fp32 for the scalar gate; k / g and b in fp32 and
    the per-row gates for the diagonal gate) is this implementation's representation, not the
    method's bytes, so it is reported apart as `side` and left out of `total`. A chunk of T
    tokens reads and writes the packed state once: 1/T of it per request-step."""
    esz = 2 if wl.io_dtype == W.IO_BF16 else 4
    H, dk, dv = wl.n_heads, wl.d_k, wl.d_v
    io = H * (2 * dk + dv) * esz + H * wl.alpha_width * 4 + H * 4 + H * dv * 4 + 4
    if wl.tokens > 1:
        state, side = 2 * slot_bytes / wl.tokens, 0
    elif wl.window <= 1:
        state, side = 2 * slot_bytes, 0
    else:
        Wn = wl.window
        state = slot_bytes + slot_bytes / Wn
        diag = wl.gate == W.GATE_DIAG
        head = 16 + (4 * dk if diag else 0)  # header (count; scalar gate: g), diagonal: g [d_k]
        kpart = 4 * dk if diag else (dk * esz + 15) // 16 * 16
        term = kpart + 4 * dv
        # per head and window: token t reads the header and t terms; tokens 0..W-2 write a
        # term and the header (count and gate(s)); the last token folds and clears the count
        reads = sum(head + t * term for t in range(Wn))
        writes = (Wn - 1) * (dk * (4 if diag else esz) + 4 * dv + (4 + 4 * dk if diag else 8)) + 4
        side = H * (reads + writes) / Wn
    return {"state": state, "side": side, "io": io, "total": state + io}


def peaks() -> tuple[float, str]:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# The sources each timed kernel is built from (its translation units, the headers they include
# and the host code that lays out its tables and launches it).
_COMMON = ["sq_step.cuh", "sq_pair.cuh", "sq_device.cuh", "sq_tile.cuh", "sq_internal.h",
           "sq_api.cu"]
KERNEL_SOURCES = {
    "k_decode": ["sq_decode.cu"] + _COMMON,
    "k_window": ["sq_window_step.cu", "sq_fold.cuh"] + _COMMON,
    "k_chunk": ["sq_chunk.cu", "sq_fold.cuh"] + _COMMON,
    "k_decode_k_quantize": ["sq_decode.cu", "sq_quant.cu"] + _COMMON,
}


def _code_only(text: str) -> str:
    """The source without comments and with whitespace collapsed: edits to comments do not
    change what the kernel computes."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_digest(kernel: str = "k_decode", root: str = ROOT) -> str:
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(root, "bit_recurrent_state_gated_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "k_decode"):
    """DRAM bytes per launch of the timed kernel from the committed ncu summary, if it was
    taken on the current source of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(p):
        return None
    digest = source_digest(kernel)
    with open(p) as f:
        for line in f:
            if line.startswith("bench-traffic:"):
                parts = dict(kv.split("=") for kv in line.split(":", 1)[1].split())
                if parts.get("source") == digest:
                    return float(parts["bytes_per_launch"])
    return None


# ---- clocks ------------------------------------------------------------------------------------

class ClockSampler:
    """Polls the SM clock and the throttle reasons through NVML while the timed region runs."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _handle(self, idx):
        import torch
        nv = self.nv
        try:
            p = torch.cuda.get_device_properties(idx)
            bus = "%08X:%02X:%02X.0" % (int(p.pci_domain_id), int(p.pci_bus_id),
                                         int(p.pci_device_id))
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[idx]) if vis and vis.split(",")[idx].isdigit() else idx
            return nv.nvmlDeviceGetHandleByIndex(phys)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, const in self.REASONS.items():
                    if r & int(getattr(nv, const, 0)):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---- CPU oracle (baseline and reference arm) ----------------------------------------------------

class OracleSample:
    """A bounded sample of the workload for the CPU oracle: the first few requests of the batch
    (all heads) in an oracle pool, with a few steps of inputs, stepped on demand."""

    def __init__(self, wl: W.Workload, t0: int = 0):
        import oracle
        self.threads = oracle.default_threads()
        self.n_req = max(1, min(wl.batch, self.threads))
        # a chunk of T tokens is the windowed oracle with W = T (requantized after the T-th token)
        window = wl.tokens if wl.tokens > 1 else wl.window
        lay = oracle.Layout(wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.fit_iters, window,
                            wl.n_outliers)
        self.pool = oracle.Pool(lay, wl.bits(), self.n_req)
        self.step = self.pool.window_step if window > 1 else self.pool.decode_step
        self.si = np.arange(self.n_req, dtype=np.int32)
        self.S0 = wl.initial_state(wl.slot_idx()[:self.n_req])
        self.pool.quantize(self.si, self.S0)
        self.horizon = rollout_calls(wl)
        self.sets = []
        for t in range(t0, t0 + max(4, wl.tokens)):
            x = wl.step_inputs(t)
            self.sets.append({k: np.ascontiguousarray(v[:self.n_req]) for k, v in x.items()})
        self.calls = 0

    def run(self, seconds: float):
        """Step until `seconds` of oracle time (at least one call): (request-steps, seconds)."""
        done, busy = 0, 0.0
        while busy < seconds or done == 0:  # only the oracle's own calls are timed
            if self.calls and self.calls % self.horizon == 0:  # a fresh rollout (untimed)
                self.pool.quantize(self.si, self.S0)
            xs = self.sets[self.calls % len(self.sets)]
            ts = time.perf_counter()
            self.step(self.si, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"],
                      threads=self.threads)
            busy += time.perf_counter() - ts
            done += self.n_req
            self.calls += 1
        return done, busy

    def describe(self, wl: W.Workload) -> str:
        return f"{self.n_req} requests x {wl.n_heads} heads"


def oracle_rate(wl: W.Workload, seconds: float, t0: int = 0):
    """Request-steps/s of the CPU oracle on a bounded sample of the workload."""
    sample = OracleSample(wl, t0)
    done, busy = sample.run(seconds)
    return done / busy, sample.threads, f"{sample.describe(wl)}, {sample.calls} steps"


# ---- GPU arm -----------------------------------------------------------------------------------

def rollout_calls(wl: W.Workload) -> int:
    """Calls in one rollout of the workload (its `steps` tokens). Runs longer than that restart
    from the initial states, outside the timed steps: the synthetic inputs cycle through a few
    seeded sets, and over thousands of steps that periodic forcing drives the 2-bit heads of
    the quantized recurrence out of range (seen in the oracle after about 1,700 steps of the
    pool workload), which is no longer the workload."""
    return max(1, wl.steps // wl.tokens)


def cold_window(wl, pool, si):
    """W tokens from the cold start (W - 1 in-window tokens, then the fold), untimed."""
    import torch
    if wl.window <= 1:
        raise SystemExit("--cold-window needs a windowed workload")
    out = torch.empty((wl.batch, wl.n_heads, wl.d_v), dtype=torch.float32, device="cuda")
    for t in range(wl.window):
        x = wl.step_inputs(t)
        if wl.io_dtype == W.IO_BF16:
            q, k, v = (torch.from_numpy(x[n + "_bf16"]).view(torch.bfloat16).cuda() for n in "qkv")
        else:
            q, k, v = (torch.from_numpy(x[n]).cuda() for n in "qkv")
        pool.decode_step(si, q, k, v, torch.from_numpy(x["alpha"]).cuda(),
                         torch.from_numpy(x["beta"]).cuda(), out)
    torch.cuda.synchronize()
    st, flag = pool.status()
    if st != 0:
        raise RuntimeError(f"device flag {flag}")
    return None


def run_ours(args, info):
    import torch

    from bit_recurrent_state_gated_b200 import sq

    dev = info.local_rank
    torch.cuda.set_device(dev)
    base = W.WORKLOADS[args.workload]
    wl = base.scaled(seed=base.seed + 1000 * info.rank)  # each rank: its own requests
    lay = sq.Layout(wl.slots, wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.io_dtype,
                    wl.fit_iters, wl.window, wl.n_outliers)
    bits = wl.bits()
    pool = sq.StatePool(lay, bits, wl.pivot_mask())
    si_np = wl.slot_idx()
    si = torch.from_numpy(si_np).cuda()
    S0_dev = [torch.from_numpy(wl.initial_state(si_np[c:c + 64])).cuda()
              for c in range(0, wl.batch, 64)]  # initial states, kept for restarts

    def restart(p, slots):  # the initial packed states again (quantized on the GPU in chunks)
        for n, c in enumerate(range(0, wl.batch, 64)):
            p.quantize(slots[c:c + 64], S0_dev[n])

    restart(pool, si)
    if args.cold_window:
        return cold_window(wl, pool, si)
    horizon = rollout_calls(wl)
    since = [0, 0]  # calls on the pool since its last restart; restarts so far

    def maybe_restart():  # untimed, like the L2 flush
        if since[0] == horizon:
            restart(pool, si)
            since[0] = 0
            since[1] += 1
        since[0] += 1
    T = wl.tokens
    n_sets = max(1, min(args.steps + args.warmup, 8))
    sets_host, sets_dev = [], []
    for t in range(n_sets):
        x = wl.chunk_inputs(t * T, T) if T > 1 else wl.step_inputs(t)
        if wl.io_dtype == W.IO_BF16:
            qkv = [torch.from_numpy(x[n + "_bf16"]).view(torch.bfloat16) for n in "qkv"]
        else:
            qkv = [torch.from_numpy(x[n]) for n in "qkv"]
        host = [a.pin_memory() for a in qkv + [torch.from_numpy(x["alpha"]),
                                               torch.from_numpy(x["beta"])]]
        sets_host.append(host)
        sets_dev.append([a.cuda() for a in host])
    out = torch.empty((wl.batch, wl.n_heads) + ((T,) if T > 1 else ()) + (wl.d_v,),
                      dtype=torch.float32, device="cuda")
    out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    sink = torch.empty(1, dtype=torch.float32, device="cuda")

    class _Flush:  # write then read a buffer twice the size of L2: L2 holds only clean lines
        @staticmethod
        def zero_():
            flush_buf.zero_()
            torch.sum(flush_buf, dim=0, keepdim=True, out=sink)

    flush = _Flush()
    stream = torch.cuda.current_stream()
    st_handle = stream.cuda_stream

    staging = side = None
    if wl.side_stream:
        staging = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32,
                              device="cuda")
        side = torch.cuda.Stream()

    def call(q, k, v, a, b, si_ptr=None, out_ptr=None):
        si_ptr = si.data_ptr() if si_ptr is None else si_ptr
        out_ptr = out.data_ptr() if out_ptr is None else out_ptr
        if wl.side_stream:
            sq.sq_decode_step_split(pool.handle, si_ptr, wl.batch, q, k, v, a, b, out_ptr,
                                    staging.data_ptr(), st_handle, side.cuda_stream)
            stream.wait_stream(side)  # the step ends when the requantization has
        elif T > 1:
            sq.sq_decode_chunk(pool.handle, si_ptr, wl.batch, T, q, k, v, a, b, out_ptr,
                               st_handle)
        else:
            sq.sq_decode_step(pool.handle, si_ptr, wl.batch, q, k, v, a, b, out_ptr, st_handle)

    def step(t):
        call(*(x.data_ptr() for x in sets_dev[t % n_sets]))

    log(f"pool ready: {wl.slots} slots x {pool.slot_bytes} B; warm-up")
    for t in range(args.warmup):
        maybe_restart()
        flush.zero_()
        step(t)
    torch.cuda.synchronize()
    st, flag = pool.status()
    if st != sq.SQ_OK:
        raise RuntimeError(f"device flag {flag} after warm-up")

    # RUNS timed regions of exactly K steps each; every region is bracketed by a barrier and a
    # device synchronization, its device time is the sum of its steps' CUDA-event times (the L2
    # flush before each step is outside the events), the max over ranks; the median region counts
    runs = max(1, args.runs)
    run_ms, run_kernel_ms = [], []
    with ClockSampler(dev, period_s=0.0005) as clocks:
        run_restarts = []
        for r in range(runs):
            restarts0 = since[1]
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            dist.barrier()
            torch.cuda.synchronize()
            for t in range(args.steps):
                maybe_restart()  # past one rollout of the workload: a fresh one (untimed)
                flush.zero_()  # every timed step starts with a cold L2
                ev[t][0].record(stream)
                step(args.warmup + r * args.steps + t)
                ev[t][1].record(stream)
            torch.cuda.synchronize()
            dist.barrier()
            kms = [a.elapsed_time(b) for a, b in ev]
            run_kernel_ms.append(kms)
            run_restarts.append(since[1] - restarts0)
            run_ms.append(dist.max_over_ranks(sum(kms), device="cuda"))
    st, flag = pool.status()
    if st != sq.SQ_OK:
        raise RuntimeError(f"device flag {flag} in the timed regions")
    log("timed regions done")
    med = sorted(range(runs), key=lambda i: run_ms[i])[runs // 2]
    dev_ms = run_ms[med]
    kernel_ms = run_kernel_ms[med]

    # end to end, through the same public calls: every step copies its q, k, v, alpha, beta from
    # pinned host memory (back to back, 256-byte aligned, one copy) and reads its o back into
    # pinned host memory. The copies run on their own streams, double-buffered, so step t+1's
    # inputs cross while step t computes and step t's o crosses while step t+1 computes. L2:
    # the steps rotate over E2E_SETS disjoint groups of slots (the batch's states, copied), so a
    # group's state has left L2 before it is stepped again.
    offs, total = [], 0
    for a in sets_host[0]:
        offs.append(total)
        total += (a.numel() * a.element_size() + 255) // 256 * 256
    packed_host = []
    for host in sets_host:
        buf = torch.empty(total, dtype=torch.uint8).pin_memory()
        for o, a in zip(offs, host):
            buf[o:o + a.numel() * a.element_size()].copy_(a.reshape(-1).view(torch.uint8))
        packed_host.append(buf)
    state_set = wl.slots * pool.slot_bytes
    n_rot = max(2, -(-2 * L2_BYTES // state_set))  # >= 2 L2s of state between reuses
    n_rot = min(n_rot, E2E_SETS)
    pool.close()
    lay_r = sq.Layout(wl.slots * n_rot, wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate,
                      wl.io_dtype, wl.fit_iters, wl.window, wl.n_outliers)
    pool = sq.StatePool(lay_r, bits, wl.pivot_mask())
    si_rot = []
    for r in range(n_rot):
        si_r = torch.from_numpy(si_np + r * wl.slots).cuda()
        restart(pool, si_r)
        si_rot.append(si_r)
    del S0_dev
    # each group stays within one rollout of the workload: at most `horizon` timed steps each
    n_e2e = min(args.steps, horizon * n_rot)
    d_in = [torch.empty(total, dtype=torch.uint8, device="cuda") for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    outs_host = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def issue_h2d(t):
        i = t % 2
        if t >= 2:
            h2d_s.wait_event(ev_comp[i])  # step t-2 has finished reading d_in[i]
        with torch.cuda.stream(h2d_s):
            d_in[i].copy_(packed_host[(args.warmup + t) % n_sets], non_blocking=True)
        ev_in[i].record(h2d_s)

    def e2e_run(n):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        h2d_s.wait_event(start)
        issue_h2d(0)
        for t in range(n):
            i = t % 2
            if t + 1 < n:
                issue_h2d(t + 1)
            stream.wait_event(ev_in[i])
            if t >= 2:
                stream.wait_event(ev_out[i])  # step t-2's o has left outs[i]
            base = d_in[i].data_ptr()
            call(*(base + o for o in offs), si_ptr=si_rot[t % n_rot].data_ptr(),
                 out_ptr=outs[i].data_ptr())
            ev_comp[i].record(stream)
            d2h_s.wait_event(ev_comp[i])
            with torch.cuda.stream(d2h_s):
                outs_host[i].copy_(outs[i], non_blocking=True)
            ev_out[i].record(d2h_s)
        stream.wait_stream(h2d_s)
        stream.wait_stream(d2h_s)
        end.record(stream)
        return start, end

    e2e_run(args.warmup)
    dist.barrier()
    torch.cuda.synchronize()
    start, end = e2e_run(n_e2e)
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = dist.max_over_ranks(start.elapsed_time(end), device="cuda")
    st, flag = pool.status()
    if st != sq.SQ_OK:
        raise RuntimeError(f"device flag {flag} in the end-to-end region")
    h2d = total
    d2h = outs_host[0].numel() * outs_host[0].element_size()

    total_req_steps = wl.batch * T * args.steps * info.world
    ab = algorithmic_bytes(wl, pool.slot_bytes)
    mean_launch_s = statistics.mean(kernel_ms) / 1e3
    achieved = ab["total"] * wl.batch * T / mean_launch_s / 1e9
    peak, peak_kind = peaks()
    kernel = ("k_chunk" if T > 1 else "k_window" if wl.window > 1 else
              "k_decode_k_quantize" if wl.side_stream else "k_decode")
    traffic = profiled_traffic(args.workload, kernel)
    res = {
        "metric": METRIC,
        "value": total_req_steps / (dev_ms / 1e3),
        "unit": UNIT,
        "n_gpus": info.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dev_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; no dataset)",
        "config": {
            "workload": f"{wl.name}: {wl.notes}",
            "batch_per_gpu": wl.batch, "heads": wl.n_heads, "d_k": wl.d_k, "d_v": wl.d_v,
            "slots_per_gpu": wl.slots, "gate": "scalar" if wl.gate == 0 else "diagonal",
            "io": "bf16" if wl.io_dtype == W.IO_BF16 else "f32", "fit_iters": wl.fit_iters,
            "state_bytes_per_request": pool.slot_bytes,
            "algorithmic_bytes_per_request_step": ab["total"],
            "side_state_bytes_per_request_step": ab["side"],
            "window": wl.window, "compensation_entries_per_head": wl.n_outliers,
            "tokens_per_call": T,
            "side_stream_split": wl.side_stream,
            "l2": "flushed before every timed step (write, then read, 256 MB)",
            "parallelism": f"dp{info.world} (requests partitioned, no collective)",
        },
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": kernel,
                     "frac_of_nominal": {"peak": NOMINAL_HBM_GBS, "frac": achieved / NOMINAL_HBM_GBS,
                                         "note": "nominal 8 TB/s HBM3e, context only"},
                     "mean_launch_us": mean_launch_s * 1e6,
                     "achieved_with_side_state": (ab["total"] + ab["side"]) * wl.batch * T
                     / mean_launch_s / 1e9 if ab["side"] else None},
        "timing": {"regions": runs, "steps_per_region": args.steps,
                   "region_ms": [round(x, 6) for x in run_ms], "reported": "median region"},
        "e2e": {"value": wl.batch * T * n_e2e * info.world / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": n_e2e, "ms_per_step": e2e_ms / n_e2e,
                "l2": f"steps rotate over {n_rot} disjoint slot groups "
                      f"({n_rot * state_set / 2**20:.0f} MiB of state)",
                "copies": "own streams, double-buffered (inputs of step t+1 and o of step t "
                          "cross while step t / t+1 computes)"},
        # per timed region: the steps' kernels, and the quantize launches of any restart between
        # steps (outside the steps' events)
        "gpu_launches": args.steps * (2 if wl.side_stream else 1)
        + run_restarts[med] * len(range(0, wl.batch, 64)),
        "rollout": {"restart_every_calls": horizon, "restarts_in_reported_region": run_restarts[med]},
        "clocks": clocks.summary(),
    }
    log("end-to-end region done")
    if info.world == 1 and info.rank == 0:
        rate, cores, sample = oracle_rate(wl, args.cpu_seconds)
        log("cpu baseline done")
        res["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample}
    pool.close()
    return res


def run_reference(args, info):
    """The CPU oracle as the reference arm, on the same workload and metric."""
    if info.rank != 0:
        return None
    wl = W.WORKLOADS[args.workload]
    # every step a bounded sample, sized so the whole run stays within about 150 s of oracle time
    per_step = max(0.02, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    sample = OracleSample(wl)
    for _ in range(args.warmup):
        sample.run(per_step)
    done = busy = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        d, b = sample.run(per_step)
        done, busy = done + d, busy + b
    el = time.perf_counter() - t0
    value = done / busy
    cores = sample.threads
    sample_txt = f"{sample.describe(wl)}, about {per_step:.3g} s of oracle time"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": info.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / max(args.steps, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 update, f32 state",
        "data": "synthetic (seeded; no dataset)",
        "config": {"workload": f"{wl.name}: {wl.notes}", "batch_per_gpu": wl.batch,
                   "heads": wl.n_heads, "d_k": wl.d_k, "d_v": wl.d_v},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"per step: {sample_txt}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def log(msg: str):
    sys.stderr.write(f"[bench {time.strftime('%H:%M:%S')}] {msg}\n")
    sys.stderr.flush()


def main():
    import faulthandler
    faulthandler.enable()
    args = parse()
    info = dist.rank_info()
    if args.impl == "reference":
        res = run_reference(args, info)
    else:
        dist.init("nccl")
        try:
            res = run_ours(args, info)
        finally:
            dist.finalize()
    if res is not None and info.rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
