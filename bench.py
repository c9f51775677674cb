"""Benchmark of the exact-attention hot path on B200.

One step = one forward pass of bf16 non-causal multi-head attention over the
seq_len sweep of the Phase 08 page's Lab 01 benchmark (B=2, H=16, d=128,
N = 512, 1024, 2048, 4096, 8192), on synthetic N(0,1) inputs resident in HBM.
L2 is flushed (a 256 MiB write) before every launch and the flush is outside the
per-launch CUDA-event pairs that give the kernel time.

The JSON line also carries, measured in the same run:
  * ``components``: causal N=8192 (H=32), GQA causal N=4096 (B=4, Hq=32,
    Hkv=8) prefill TFLOP/s, and the paged GQA decode (64 sequences, context
    U[512, 8192], 16-token pages) in HBM GB/s over a bf16 cache and over 8-bit
    (E4M3, INT8) caches of the same shape, each as a fraction of the measured
    peak; the chunked prefill over the paged cache (16 sequences, a 512-token
    chunk after U[0, 7680] cached tokens) in TFLOP/s; and the backward (dQ,
    dK, dV) of the N=8192 MHA and causal workloads in TFLOP/s of the
    algorithm's five products.  Each component is the median of its flushed
    launches (the mean is kept beside it as ``ms_mean``);
  * ``roofline`` for the prefill kernel (tensor-bound);
  * ``e2e``: the same sweep through the public API with pinned host buffers,
    host->device and device->host copies inside the timed region;
  * ``cpu_baseline``: the fp64 CPU oracle timed on a bounded sample.

``--impl reference`` times the CPU oracle on the same workload instead (a few
heads per step, all host cores), as the reference arm.
Multi-GPU (torchrun): every rank runs the whole workload on its own GPU (the
path needs no collective); value = work of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_101_b200 import synthetic as syn  # noqa: E402

METRIC = "attention fwd TFLOP/s (bf16, causal/non) & decode HBM GB/s, % of roofline"
WORKLOAD = "bf16 MHA non-causal prefill sweep B=2 H=16 d=128 N=512..8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest(name: str) -> str:
    with open(os.path.join(ROOT, "exact_io_aware_101_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(summary: str, kernel_src: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the source."""
    path = os.path.join(ROOT, "profiles", summary)
    try:
        text = open(path).read()
    except OSError:
        return None
    m_src = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_src or not m_b or m_src.group(1) != source_digest(kernel_src):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, polled through NVML about every
    millisecond while the timed region runs (nvidia-smi's 200 ms period is longer
    than a short timed region).  Read-only: no clock or power setting is touched."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
        for cand in (uuid, "GPU-" + uuid):
            try:
                return pynvml.nvmlDeviceGetHandleByUUID(cand)
            except Exception:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _run(self, h):
        import pynvml
        while not self._stop.is_set():
            try:
                mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, reasons))
            except Exception:
                break
            time.sleep(0.001)

    def __enter__(self):
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(h,), daemon=True)
            self._thread.start()
            time.sleep(0.003)
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None
        import pynvml
        mhz = sorted(m for m, _ in self.samples)
        active = set()
        for _, bits in self.samples:
            for name, const in self.REASONS:
                if bits & getattr(pynvml, const, 0):
                    active.add(name)
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(mhz), "source": "nvml"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over all ranks (CUDA-event times are per rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(work_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return work_per_rank * world / max_seconds


# ------------------------------------------------------------ GPU workloads
class Prefill:
    def __init__(self, cfg, lib):
        self.cfg = cfg
        self.lib = lib
        self.q, self.k, self.v = syn.prefill_inputs(cfg, device="cuda")
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(cfg.B, cfg.Hq, cfg.N, dtype=torch.float32, device="cuda")
        self.slopes = torch.tensor(syn.alibi_slopes(cfg.Hq), dtype=torch.float32, device="cuda")

    def launch(self):
        c = self.cfg
        if c.window or c.alibi:
            rc = self.lib.attn_fwd_ext(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                       self.o.data_ptr(), self.lse.data_ptr(), c.B, c.Hq, c.Hkv,
                                       c.N, c.d, c.scale, int(c.causal), c.window,
                                       self.slopes.data_ptr() if c.alibi else None,
                                       torch.cuda.current_stream().cuda_stream)
        else:
            rc = self.lib.attn_fwd(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                   self.o.data_ptr(), self.lse.data_ptr(), c.B, c.Hq, c.Hkv, c.N,
                                   c.d, c.scale, int(c.causal),
                                   torch.cuda.current_stream().cuda_stream)
        if rc != 0:
            raise RuntimeError("attn_fwd failed: %d" % rc)
        return 1  # kernels launched


class Decode:
    def __init__(self, cfg, lib):
        import exact_io_aware_101_b200 as ea
        self.cfg = cfg
        self.lib = lib
        self.inp = syn.decode_inputs(cfg, device="cuda")
        self.o = torch.empty_like(self.inp["q"])
        self.lse = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
        self.ws_bytes = ea.decode_workspace_bytes(cfg.S, cfg.Hq, cfg.d, cfg.max_blocks)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.bytes = syn.decode_bytes(self.inp["seq_lens"].cpu().tolist(), cfg.Hkv, cfg.d, cfg.Hq,
                                      cfg.page_size)

    def launch(self):
        c, i = self.cfg, self.inp
        rc = self.lib.attn_decode_paged(
            i["q"].data_ptr(), i["k_pages"].data_ptr(), i["v_pages"].data_ptr(),
            i["block_table"].data_ptr(), i["seq_lens"].data_ptr(), self.o.data_ptr(),
            self.lse.data_ptr(), c.S, c.Hq, c.Hkv, c.d, c.page_size, c.max_blocks, c.num_pages,
            c.scale, self.ws.data_ptr(), self.ws_bytes, torch.cuda.current_stream().cuda_stream)
        if rc != 0:
            raise RuntimeError("attn_decode_paged failed: %d" % rc)
        return 2  # split + combine


class Backward:
    """Backward of a prefill workload: the forward's O and L are computed once
    (outside the timing), dO is N(0,1); one launch = prep + dK/dV + dQ kernels.
    FLOPs: the algorithm's five N x N x d products, 10 * B * Hq * N^2 * d
    (half for causal), not the seven this implementation spends."""

    def __init__(self, cfg, lib):
        import exact_io_aware_101_b200 as ea
        self.cfg = cfg
        self.lib = lib
        self.q, self.k, self.v = syn.prefill_inputs(cfg, device="cuda")
        g = torch.Generator(device="cuda")
        g.manual_seed(cfg.seed + 7)
        self.do = torch.randn(self.q.shape, generator=g, device="cuda").to(torch.bfloat16)
        self.o, self.lse = ea.attn_fwd(self.q, self.k, self.v, causal=cfg.causal)
        self.dq = torch.empty_like(self.q)
        self.dk = torch.empty_like(self.k)
        self.dv = torch.empty_like(self.v)
        self.ws_bytes = ea.bwd_workspace_bytes(cfg.B, cfg.Hq, cfg.N)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.flops = 2.5 * cfg.flops

    def launch(self):
        c = self.cfg
        rc = self.lib.attn_bwd(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                               self.o.data_ptr(), self.lse.data_ptr(), self.do.data_ptr(),
                               self.dq.data_ptr(), self.dk.data_ptr(), self.dv.data_ptr(), c.B, c.Hq,
                               c.Hkv, c.N, c.d, c.scale, int(c.causal), 0, None, self.ws.data_ptr(),
                               self.ws_bytes, torch.cuda.current_stream().cuda_stream)
        if rc != 0:
            raise RuntimeError("attn_bwd failed: %d" % rc)
        return 3  # prep + dK/dV + dQ


class ChunkedPrefill:
    """Chunked prefill over the paged cache (the CHUNKED workload)."""

    def __init__(self, cfg, lib):
        self.cfg, self.lib = cfg, lib
        self.inp = syn.chunked_inputs(cfg, device="cuda")
        i = self.inp
        self.T = int(i["q"].shape[0])
        self.o = torch.empty_like(i["q"])
        self.lse = torch.empty(self.T, cfg.Hq, dtype=torch.float32, device="cuda")
        self.num_pages = int(i["k_pages"].shape[0])
        self.flops = syn.chunked_flops(i["seq_lens"].cpu().tolist(), i["cu_q"].cpu().tolist(),
                                       cfg.Hq, cfg.d)

    def launch(self):
        c, i = self.cfg, self.inp
        rc = self.lib.attn_prefill_paged(
            i["q"].data_ptr(), i["k_pages"].data_ptr(), i["v_pages"].data_ptr(),
            i["block_table"].data_ptr(), i["seq_lens"].data_ptr(), i["cu_q"].data_ptr(),
            self.o.data_ptr(), self.lse.data_ptr(), c.S, c.Hq, c.Hkv, self.T, c.qlen, c.d,
            c.page_size, c.max_blocks, self.num_pages, c.scale, 0, None,
            torch.cuda.current_stream().cuda_stream)
        if rc != 0:
            raise RuntimeError("attn_prefill_paged failed: %d" % rc)
        return 1


class DecodeQ8:
    """The decode workload over an 8-bit cache (same q, lengths and placement)."""

    def __init__(self, cfg, lib, fmt):
        import exact_io_aware_101_b200 as ea
        self.cfg, self.lib, self.fmt = cfg, lib, fmt
        self.code = ea.KV_FORMATS[fmt]
        self.inp = syn.decode_inputs_q8(cfg, fmt=fmt, device="cuda")
        self.o = torch.empty_like(self.inp["q"])
        self.lse = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
        self.ws_bytes = ea.decode_workspace_bytes(cfg.S, cfg.Hq, cfg.d, cfg.max_blocks)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.bytes = syn.decode_bytes(self.inp["seq_lens"].cpu().tolist(), cfg.Hkv, cfg.d, cfg.Hq,
                                      cfg.page_size, kv_elem_bytes=1)

    def launch(self):
        c, i = self.cfg, self.inp
        rc = self.lib.attn_decode_paged_q8(
            i["q"].data_ptr(), i["k_pages"].data_ptr(), i["v_pages"].data_ptr(),
            i["k_scales"].data_ptr(), i["v_scales"].data_ptr(), self.code,
            i["block_table"].data_ptr(), i["seq_lens"].data_ptr(), self.o.data_ptr(),
            self.lse.data_ptr(), c.S, c.Hq, c.Hkv, c.d, c.page_size, c.max_blocks, c.num_pages,
            c.scale, self.ws.data_ptr(), self.ws_bytes, torch.cuda.current_stream().cuda_stream)
        if rc != 0:
            raise RuntimeError("attn_decode_paged_q8 failed: %d" % rc)
        return 2  # split + combine


def timed_launches(items, flush, reps):
    """Per-item list of CUDA-event durations (ms), L2 flushed before each launch."""
    times = [[] for _ in items]
    launches = 0
    for _ in range(reps):
        for idx, it in enumerate(items):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            launches += it.launch()
            e1.record()
            times[idx].append((e0, e1))
    torch.cuda.synchronize()
    return [[a.elapsed_time(b) for a, b in row] for row in times], launches


def timed_component(items, flush, reps):
    """A component's 3 warm-up launches, then its timed launches with the SM clock
    sampled meanwhile (a component that follows a heavy one may run while power
    capping holds the clock down).  Returns the durations and the clock summary,
    reduced to the median clock and the reasons seen."""
    timed_launches(items, flush, 3)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t, _ = timed_launches(items, flush, reps)
    c = clk.summary()
    return t, ({"sm_mhz": c["sm_mhz"], "reasons": c["reasons"]} if c else None)


def component_time(ms_list):
    """Median (seconds) and mean (ms) of one component's flushed launch times: the
    median is the reported figure, robust to a slow launch while clocks or power
    settle after the previous component; the mean is kept beside it."""
    ts = sorted(ms_list)
    n = len(ts)
    med = ts[n // 2] if n % 2 else 0.5 * (ts[n // 2 - 1] + ts[n // 2])
    return med / 1e3, sum(ts) / n


def e2e_sweep(items, reps):
    """The sweep through the public API with pinned host buffers (H2D + call + D2H).

    Every step copies each workload's q, k, v from pinned host memory, calls
    attn_fwd on them and reads O and L back into pinned host memory.  The
    copies in, the calls and the copies out run on three streams ordered by
    events, so one workload's copy overlaps the previous one's kernel and the
    read-back before that (host-device copies in both directions share the
    link at once).  The event pair brackets all three streams."""
    import exact_io_aware_101_b200 as ea
    host = []
    for it in items:
        host.append(dict(q=it.q.cpu().pin_memory(), k=it.k.cpu().pin_memory(),
                         v=it.v.cpu().pin_memory(), o=torch.empty(it.o.shape, dtype=it.o.dtype).pin_memory(),
                         l=torch.empty(it.lse.shape, dtype=torch.float32).pin_memory()))
    h2d = sum(h["q"].nbytes + h["k"].nbytes + h["v"].nbytes for h in host)
    d2h = sum(h["o"].nbytes + h["l"].nbytes for h in host)
    dev = [dict(q=torch.empty_like(it.q), k=torch.empty_like(it.k), v=torch.empty_like(it.v))
           for it in items]
    s_run = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in items]
    ev_run = [torch.cuda.Event() for _ in items]
    ran = [False] * len(items)

    def once():
        for i, (it, h, d) in enumerate(zip(items, host, dev)):
            if ran[i]:
                s_in.wait_event(ev_run[i])  # the last call on these buffers is done
            with torch.cuda.stream(s_in):
                d["q"].copy_(h["q"], non_blocking=True)
                d["k"].copy_(h["k"], non_blocking=True)
                d["v"].copy_(h["v"], non_blocking=True)
                ev_in[i].record(s_in)
            s_run.wait_event(ev_in[i])
            o, l = ea.attn_fwd(d["q"], d["k"], d["v"], causal=it.cfg.causal, scale=it.cfg.scale)
            ev_run[i].record(s_run)
            s_out.wait_event(ev_run[i])
            with torch.cuda.stream(s_out):
                h["o"].copy_(o, non_blocking=True)
                h["l"].copy_(l, non_blocking=True)
            o.record_stream(s_out)
            l.record_stream(s_out)
            ran[i] = True

    once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_run)
    s_in.wait_stream(s_run)
    s_out.wait_stream(s_run)
    for _ in range(reps):
        once()
    s_run.wait_stream(s_in)
    s_run.wait_stream(s_out)
    e1.record(s_run)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps, h2d, d2h


def cpu_oracle_sample(target_s=10.0):
    """Time the fp64 oracle on whole (batch, head) slices of the N=8192 MHA workload."""
    import oracle
    cfg = syn.MHA_SWEEP[4]
    q, k, v = syn.prefill_inputs(cfg)
    BH = cfg.B * cfg.Hq
    qf = q.float().reshape(1, BH, cfg.N, cfg.d).numpy()
    kf = k.float().reshape(1, BH, cfg.N, cfg.d).numpy()
    vf = v.float().reshape(1, BH, cfg.N, cfg.d).numpy()
    threads = oracle.max_threads()
    heads = 1
    while True:
        t0 = time.perf_counter()
        oracle.attention(qf[:, :heads], kf[:, :heads], vf[:, :heads], scale=cfg.scale)
        elapsed = time.perf_counter() - t0
        if elapsed >= target_s or heads >= BH:
            break
        heads = min(BH, max(heads + 1, int(heads * target_s / max(elapsed, 1e-3)) + 1))
    flops = 4.0 * heads * cfg.N * cfg.N * cfg.d
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": "fp64 oracle (materialised S, two-pass softmax) on %d (batch, head) slice(s) "
                      "of the N=8192 MHA workload: %.1f GFLOP in %.2f s"
                      % (heads, flops / 1e9, elapsed)}


# --------------------------------------------------------------- arms
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    threads = oracle.max_threads()
    data = []
    for cfg in syn.MHA_SWEEP:
        q, k, v = syn.prefill_inputs(cfg)
        data.append((cfg, q[:1, :1].float().numpy(), k[:1, :1].float().numpy(),
                     v[:1, :1].float().numpy()))

    def step():
        for cfg, q, k, v in data:
            oracle.attention(q, k, v, scale=cfg.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    flops = sum(4.0 * c.N * c.N * c.d for c, *_ in data)
    value = flops / dt / 1e12
    sample = ("fp64 CPU oracle, one (batch, head) of each N in the sweep per step "
              "(%.1f GFLOP per step)" % (flops / 1e9))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": "one head per N"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import exact_io_aware_101_b200 as ea
    rank, world, local = dist_setup(args)
    lib = ea.library()
    peaks, peak_kind = load_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    sweep = [Prefill(c, lib) for c in syn.MHA_SWEEP]
    sweep_flops = sum(p.cfg.flops for p in sweep)

    # warm-up, then exactly K timed steps bracketed by barrier + synchronize
    for _ in range(args.warmup):
        for p in sweep:
            flush.zero_()
            p.launch()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_wall0 = time.perf_counter()
        times, launches = timed_launches(sweep, flush, args.steps)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall0
    barrier(world)
    torch.cuda.synchronize()
    if ea.device_status() != 0:
        raise RuntimeError("device status word set during the timed region")

    kernel_s = sum(sum(row) for row in times) / 1e3
    kernel_s_max = max_over_ranks(kernel_s, world)
    value = aggregate(sweep_flops * args.steps, world, kernel_s_max) / 1e12
    ms_per_step = kernel_s_max * 1e3 / args.steps
    per_n = {p.cfg.name: p.cfg.flops / (sum(t) / len(t) / 1e3) / 1e12 for p, t in zip(sweep, times)}

    peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # Roofline of the dominant launch: the N=8192 prefill, about two thirds of a step.
    big = max(range(len(sweep)), key=lambda i: sweep[i].cfg.flops)
    big_s = sum(times[big]) / len(times[big]) / 1e3
    big_tf = sweep[big].cfg.flops / big_s / 1e12
    roofline = {"bound": "tensor", "achieved": big_tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": big_tf / peak_tf,
                "traffic": profiled_traffic("prefill_bf16_mha_n8192.md", "prefill_sm100.cu"),
                "peak_source": peak_kind + " bf16_tflops (burst)",
                "kernel": "prefill_bf16_kernel<128, 0, 0, 0> (whole pairs), %s launch (%.0f%% of the step)"
                          % (sweep[big].cfg.name, 100.0 * sum(times[big]) / sum(sum(t) for t in times)),
                "algorithmic": "4*B*H*N^2*d = %.4g FLOP per launch; %d bytes (Q,K,V read, O,L written)"
                               % (sweep[big].cfg.flops, sweep[big].cfg.bytes),
                "sweep_achieved": sweep_flops * args.steps / kernel_s / 1e12}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 2 * world, "seq_len": "512..8192",
                       "parallelism": "replicas x%d" % world,
                       "l2": "flushed before every launch (256 MiB write, outside the timing)"},
            "per_seq_len_tflops": per_n, "roofline": roofline, "gpu_launches": launches,
            "wall_s_timed_region": t_wall}
    clocks = clk.summary()
    if clocks:
        line["clocks"] = clocks

    if not args.skip_components:
        comps = {"_timing": "per component: 3 warm-up launches, then args.component_reps "
                            "launches each after an L2 flush; ms = median, ms_mean = mean; "
                            "clocks = median SM clock and throttle reasons during those launches"}
        for cfg in (syn.CAUSAL, syn.GQA, syn.WINDOW, syn.ALIBI):
            it = Prefill(cfg, lib)
            t, ck = timed_component([it], flush, args.component_reps)
            sec, mean_ms = component_time(t[0])
            tf = cfg.flops / sec / 1e12
            comps[cfg.name] = {"tflops": tf, "frac_of_peak": tf / peak_tf, "ms": sec * 1e3, "ms_mean": mean_ms,
                               "clocks": ck}
            del it
        it = ChunkedPrefill(syn.CHUNKED, lib)
        t, ck = timed_component([it], flush, args.component_reps)
        sec, mean_ms = component_time(t[0])
        tf = it.flops / sec / 1e12
        comps[syn.CHUNKED.name] = {"tflops": tf, "frac_of_peak": tf / peak_tf, "ms": sec * 1e3, "ms_mean": mean_ms,
                                   "flops": it.flops, "flops_counted": "4*d per visible pair",
                                   "clocks": ck}
        del it
        for cfg in (syn.MHA_SWEEP[-1], syn.CAUSAL):
            it = Backward(cfg, lib)
            t, ck = timed_component([it], flush, args.component_reps)
            sec, mean_ms = component_time(t[0])
            tf = it.flops / sec / 1e12
            comps["bwd_" + cfg.name] = {"tflops": tf, "frac_of_peak": tf / peak_tf,
                                        "ms": sec * 1e3, "ms_mean": mean_ms, "flops": it.flops,
                                        "flops_counted": "5 products of the algorithm (2.5x fwd)",
                                        "clocks": ck}
            del it
        dec = Decode(syn.DECODE, lib)
        t, ck = timed_component([dec], flush, args.component_reps)
        sec, mean_ms = component_time(t[0])
        torch.cuda.synchronize()
        if ea.decode_read_status(dec.ws) != 0:
            raise RuntimeError("decode status word set in the decode component")
        gbs = dec.bytes / sec / 1e9
        comps["decode_paged_gqa"] = {"gbs": gbs, "frac_of_peak": gbs / peak_hbm, "ms": sec * 1e3, "ms_mean": mean_ms,
                                     "algorithmic_bytes": dec.bytes,
                                     "peak_gbs": peak_hbm,
                                     "traffic": profiled_traffic("decode_paged_gqa.md",
                                                                 "decode_paged.cu"),
                                     "bound": "hbm", "clocks": ck}
        del dec
        for fmt in ("e4m3", "int8"):
            dq = DecodeQ8(syn.DECODE, lib, fmt)
            t, ck = timed_component([dq], flush, args.component_reps)
            sec, mean_ms = component_time(t[0])
            torch.cuda.synchronize()
            if ea.decode_read_status(dq.ws) != 0:
                raise RuntimeError("decode status word set in the %s decode component" % fmt)
            gbs = dq.bytes / sec / 1e9
            comps["decode_paged_gqa_" + fmt] = {
                "gbs": gbs, "frac_of_peak": gbs / peak_hbm, "ms": sec * 1e3, "ms_mean": mean_ms,
                "algorithmic_bytes": dq.bytes, "peak_gbs": peak_hbm,
                "traffic": profiled_traffic("decode_q8_gqa.md", "decode_q8.cu"), "bound": "hbm",
                "clocks": ck}
            del dq
        if ea.device_status() != 0:
            raise RuntimeError("device status word set in the component runs")
        line["components"] = comps

    if not args.skip_e2e:
        ms, h2d, d2h = e2e_sweep(sweep, max(1, min(args.steps, 5)))
        e2e_s = max_over_ranks(ms / 1e3, world)
        line["e2e"] = {"value": aggregate(sweep_flops, world, e2e_s) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank == 0 and world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_oracle_sample()

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_only(args):
    """Launch one workload's kernels a few times (no flush, no JSON): for ncu captures."""
    import exact_io_aware_101_b200 as ea
    torch.cuda.set_device(0)
    lib = ea.library()
    table = {c.name: c for c in syn.MHA_SWEEP + (syn.CAUSAL, syn.GQA, syn.WINDOW, syn.ALIBI)}
    q8 = {syn.DECODE.name + "_" + f: f for f in ("e4m3", "int8")}
    bwd = {"bwd_" + c.name: c for c in (syn.MHA_SWEEP[-1], syn.CAUSAL, syn.MHA_SWEEP[2])}
    if args.only in bwd:
        it = Backward(bwd[args.only], lib)
    elif args.only == syn.CHUNKED.name:
        it = ChunkedPrefill(syn.CHUNKED, lib)
    elif args.only == syn.DECODE.name:
        it = Decode(syn.DECODE, lib)
    elif args.only in q8:
        it = DecodeQ8(syn.DECODE, lib, q8[args.only])
    elif args.only in table:
        it = Prefill(table[args.only], lib)
    else:
        raise SystemExit("unknown workload %r; one of %s"
                         % (args.only, sorted(table) + [syn.DECODE.name] + sorted(q8) + sorted(bwd) + [syn.CHUNKED.name]))
    for _ in range(args.reps):
        it.launch()
    torch.cuda.synchronize()
    st = ea.device_status()
    if hasattr(it, "ws") and isinstance(it, (Decode, DecodeQ8)):
        st |= ea.decode_read_status(it.ws)
    print("ran %s x%d, device status %d" % (args.only, args.reps, st))
    return 0 if st == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--component-reps", type=int, default=10)
    ap.add_argument("--skip-components", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--only", default=None, help="profile mode: run one workload --reps times")
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args()
    if args.only:
        return run_only(args)
    if args.warmup < 3 and args.impl == "ours":
        print("note: at least 3 warm-up steps are required; using 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
