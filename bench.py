"""Benchmark of the DuoAttention hybrid-GQA attention path on B200.

Default workload (one GPU): one-token decode, B=32 sequences at context
32768, 48 query / 8 KV heads, head_dim 128, 2 of 8 KV heads full-context
(seeded mask), the other 6 streaming heads with 64 sink + 256 recent slots
and ring pointers at random offsets.  A step is one ``duo_attn_decode`` over
the whole batch.  Metric: algorithmic HBM bytes per second (K and V rows the
heads must read, plus q and out), inputs resident in HBM and larger than L2.

  python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]
                  [--workload decode_b32|prefill_16k|sliding_32k|stack40]

With N > 1 (torchrun, one process per GPU) every rank decodes its own batch
of 32 (weak scaling, no data-path collective); the time is the max over ranks.
``--impl reference`` times the float64 CPU oracle on this host's cores on a
bounded sample of the same workload, in the same unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kv_cache_reduction_b200 as duo  # noqa: E402
from kv_cache_reduction_b200 import inputs  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "decode attn HBM GB/s (% of ~8 TB/s); prefill attn TFLOP/s (% bf16 peak)"


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ distributed plumbing
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: every rank contributes its own elapsed time."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return base + 7919 * rank


def aggregate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU while a timed
    region runs.  With NVML, a thread polls back to back between begin() and
    end(), which time_steps calls around its timed region; the GPU is found
    by its PCI address, so a remapped device visibility cannot pick another
    one.  Without NVML, nvidia-smi samples every 200 ms around the region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.nv = None
        self.handle = None
        self.max_mhz = None
        self.rows = []                 # (SM MHz, clock-event reason bits) per NVML sample
        self.active = threading.Event()
        self.done = threading.Event()
        self.thread = None

    def _nvml(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            props = torch.cuda.get_device_properties(self.idx)
            want = (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            for i in range(nv.nvmlDeviceGetCount()):
                h = nv.nvmlDeviceGetHandleByIndex(i)
                pci = nv.nvmlDeviceGetPciInfo(h)
                if (pci.domain, pci.bus, pci.device) == want:
                    return nv, h
        except Exception:
            pass
        return None, None

    def __enter__(self):
        self.nv, self.handle = self._nvml()
        if self.handle is not None:
            try:
                self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
                self.thread = threading.Thread(target=self._poll, daemon=True)
                self.thread.start()
                return self
            except Exception:
                self.handle = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
            os.unlink(self.path)
            self.path = None
        return self

    def _poll(self):
        nv, h = self.nv, self.handle
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.done.is_set():
            if not self.active.is_set():
                time.sleep(0.0005)
                continue
            try:      # back to back while the region runs (each query releases the GIL)
                self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), reasons(h)))
            except Exception:
                return

    def begin(self):
        self.active.set()

    def end(self):
        self.active.clear()

    def __exit__(self, *exc):
        self.done.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.handle is not None:
            return self._nvml_summary()
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, p in rows:
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        busy = [r[0] for r in rows] or [0.0]
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons),
                "source": "nvidia-smi every 200 ms around the timed region"}

    def _nvml_summary(self):
        nv = self.nv
        masks = [(name, getattr(nv, attr, 0)) for name, attr in self.REASONS]
        idle = getattr(nv, "nvmlClocksEventReasonGpuIdle", 0)
        # samples the driver flags as idle (the region's first microseconds) are
        # left out of the median under load
        loaded = [r for r in self.rows if not (r[1] & idle)] or self.rows
        out = {"sm_mhz": statistics.median(r[0] for r in loaded) if loaded else None,
               "sm_max_mhz": self.max_mhz, "samples": len(loaded),
               "reasons": sorted({name for _, bits in self.rows for name, m in masks if bits & m}),
               "source": "NVML, polled during the timed region"}
        if not loaded:
            out["reasons"] = ["no samples"]
        return out


# ------------------------------------------------------------------ workloads
class DecodeB32:
    """One-token decode at context 32768 for 32 sequences.  With product=False
    only the inputs are built (plain torch, no call into the library), as the
    reference arm needs them."""

    def __init__(self, rank: int, product: bool = True):
        w = self.w = inputs.workload("decode_b32")
        B, n = w.batch, w.seq_len
        self.params = duo.DuoParams(B, 48, 8, 128, inputs.SINK, inputs.RECENT, 0, 128 ** -0.5,
                                    w.full_mask, None)
        seed = rank_seed(w.seed, rank)
        self.cache = duo.DuoCache.allocate(self.params, n)
        for i, t in enumerate((self.cache.full_k, self.cache.full_v, self.cache.strm_k,
                               self.cache.strm_v)):
            inputs.randn_bf16_into(t, seed * 10 + i)
        rng = np.random.default_rng(seed)
        self.cache.seq_len.fill_(n)
        self.cache.ring_head.copy_(torch.as_tensor(rng.integers(0, inputs.RECENT, size=B),
                                                   dtype=torch.int32))
        self.q = inputs.randn_bf16((B, 48, 128), seed + 5, "cuda")
        self.out = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((B, 48), dtype=torch.float32, device="cuda")
        self.ws = duo.workspace_for(self.params, n) if product else None
        self.bytes = decode_bytes(B, n, self.params.n_full, self.params.n_ring)
        self.launches_per_step = 2
        self.unit = "GB/s"
        self.kernel = "decode_split + decode_merge (one duo_attn_decode call)"
        self.traffic_key = ("decode_split", "decode_b32")

    def step(self):
        duo.duo_attn_decode(self.params, self.cache, self.q, self.w.seq_len, self.out, self.lse,
                            self.ws)

    def e2e_buffers(self):
        self.h_q = self.q.cpu().pin_memory()
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()
        self.d_q = torch.empty_like(self.q)
        return self.h_q.numel() * 2, self.h_out.numel() * 2 + self.h_lse.numel() * 4

    def e2e_step(self):
        self.d_q.copy_(self.h_q, non_blocking=True)
        duo.duo_attn_decode(self.params, self.cache, self.d_q, self.w.seq_len, self.out, self.lse,
                            self.ws)
        self.h_out.copy_(self.out, non_blocking=True)
        self.h_lse.copy_(self.lse, non_blocking=True)

    def config(self):
        return {"workload": "decode_b32: one-token decode, B=32, context 32768, 48 Q / 8 KV heads, "
                            "head_dim 128, 2 of 8 KV heads full, sink 64 + recent 256 ring",
                "batch_per_gpu": self.w.batch, "context": self.w.seq_len,
                "full_mask": list(self.w.full_mask),
                "l2": "inputs larger than L2 (1.1 GB of cache per step)"}

    # -------------------------------------------------- CPU oracle on a bounded sample
    def oracle_sample(self, budget_s: float = 15.0):
        """The oracle over whole decode steps: every (sequence, query head) row of
        the batch in one call, so that its dynamic row schedule keeps every host
        thread busy (the full heads' long rows outnumber the threads)."""
        import oracle
        p = self.params
        olayer = oracle.Layer(p.batch, 48, 8, 128, p.sink, p.recent, 0, p.softmax_scale,
                              p.full_mask, None)
        hc = oracle.Cache(olayer, self.w.seq_len)
        hc.full_k, hc.full_v = inputs.bits(self.cache.full_k), inputs.bits(self.cache.full_v)
        hc.strm_k, hc.strm_v = inputs.bits(self.cache.strm_k), inputs.bits(self.cache.strm_v)
        hc.seq_len = self.cache.seq_len.cpu().numpy().astype(np.int32)
        hc.ring_head = self.cache.ring_head.cpu().numpy().astype(np.int32)
        qb = inputs.bits(self.q)
        n = self.w.seq_len
        step_bytes = decode_bytes(p.batch, n, p.n_full, p.n_ring)
        rows = p.batch * 48
        threads = oracle.num_threads()

        def run(_):
            oracle.attn_decode(olayer, hc, qb)

        done_bytes, t_total, used = timed_sample(["step"], run, lambda _: step_bytes, budget_s)
        return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": threads,
                "threads_busy": min(threads, p.batch * p.n_full * 6), "kind": "oracle",
                "sample": f"{used} whole decode steps ({rows} rows per call, "
                          f"{p.batch * p.n_full * 6} of them full-head rows of {n} keys), "
                          f"float64, {t_total:.1f} s"}


def timed_sample(units, run, nbytes, budget_s: float, max_passes: int = 64):
    """Runs run(u) over the units in order, cycling through them, until the
    timed work reaches budget_s (at least one unit, at most max_passes passes).
    Returns (bytes the units cover, seconds spent in run, units run)."""
    done_bytes, t_total, used = 0, 0.0, 0
    while used < max_passes * len(units):
        u = units[used % len(units)]
        t0 = time.perf_counter()
        run(u)
        t_total += time.perf_counter() - t0
        done_bytes += nbytes(u)
        used += 1
        if t_total >= budget_s:
            break
    return done_bytes, t_total, used


def attended_pairs(L: int, span):
    """Number of (query, key) pairs a head attends over an L-token prefill:
    L(L+1)/2 for a full head, sum_i min(i+1, span) for a band of `span` keys."""
    if span is None:
        return L * (L + 1) // 2
    m = min(L, span)
    return m * (m + 1) // 2 + (L - m) * span


def prefill_flops(w) -> int:
    """Algorithmic FLOPs of one prefill of workload w (48 query heads, 6 per KV
    head): 4 * 128 per attended (query, key) pair and query head (QK^T and PV,
    2 * 128 each); masked tile area, padding and the sink term are not counted."""
    pairs = 0
    for g in range(8):
        span = w.window if w.window else (None if w.full_mask[g] else inputs.SINK + inputs.RECENT)
        pairs += 6 * attended_pairs(w.seq_len, span)
    return 4 * 128 * pairs * w.batch


def decode_bytes(batch: int, n: int, n_full: int, n_ring: int,
                 span: int = inputs.SINK + inputs.RECENT) -> int:
    """Algorithmic bytes of one one-token decode at context n (the query at
    position n - 1, already appended): the K and V rows (2 x 128 bf16 each) every
    KV head attends to, read once for its 6 query heads, plus q and out (48 x 128
    bf16 each per sequence).  A ring head (sink + recent, or a sliding window)
    attends min(n, span) rows."""
    rows = batch * (n_full * n + n_ring * min(n, span))
    return rows * 2 * 128 * 2 + 2 * batch * 48 * 128 * 2


def block_ring_rows(n: int, sink: int, recent: int) -> int:
    """Cached rows of one streaming head that a verify block attends to: its
    queries sit at positions n, n + 1, ... of a cache of n tokens, so the union
    of their bands is the sink plus the recent - 1 cached tokens before n (the
    first query's band reaches back the furthest)."""
    return min(n, sink) + max(0, min(n - sink, recent - 1))


def verify_bytes(batch: int, n: int, q_len: int, n_full: int, n_ring: int,
                 sink: int = inputs.SINK, recent: int = inputs.RECENT) -> int:
    """Algorithmic bytes of one verify-block decode: the cached K/V rows the
    block's queries attend to (each read once for all of them), the block's own
    K/V rows, and the block's q and out."""
    rows = batch * (n_full * n + n_ring * block_ring_rows(n, sink, recent)) + \
        batch * (n_full + n_ring) * q_len
    return rows * 2 * 128 * 2 + 2 * batch * q_len * 48 * 128 * 2


def stack_bytes(w) -> int:
    """Algorithmic bytes of one decode step through the layer stack of workload
    w: each DuoAttention layer's full and streaming heads, each sliding layer's
    window ring."""
    total = 0
    for mask in inputs.stack_layer_masks(w):
        if mask is None:
            total += decode_bytes(w.batch, w.seq_len, 0, 8, inputs.WINDOW)
        else:
            n_full = sum(1 for m in mask if m)
            total += decode_bytes(w.batch, w.seq_len, n_full, 8 - n_full)
    return total


class Stack40:
    """One decode step through the 40-layer stack: B=16 sequences at context
    131072; layers 3, 7, ..., 39 are DuoAttention layers (2 of 8 heads full),
    the other 30 sliding-window layers (window 512) with sink logits.  The 40
    decode calls are captured once in a CUDA graph and replayed per step."""

    def __init__(self, rank: int, product: bool = True):
        w = self.w = inputs.workload("stack40")
        B, n = w.batch, w.seq_len
        masks = inputs.stack_layer_masks(w)
        seed = rank_seed(w.seed, rank)
        rng = np.random.default_rng(seed)
        self.layers = []
        self.bytes = stack_bytes(w)
        max_ws = 0
        for li, mask in enumerate(masks):
            if mask is None:
                sig = inputs.randn_f32((48,), seed * 100 + li, "cuda")
                p = duo.DuoParams(B, 48, 8, 128, 0, 0, inputs.WINDOW, 128 ** -0.5, (0,) * 8, sig)
            else:
                p = duo.DuoParams(B, 48, 8, 128, inputs.SINK, inputs.RECENT, 0, 128 ** -0.5, mask, None)
            cache = duo.DuoCache.allocate(p, n)
            for i, t in enumerate((cache.full_k, cache.full_v, cache.strm_k, cache.strm_v)):
                if t is not None:
                    inputs.randn_bf16_into(t, (seed * 100 + li) * 10 + i)
            cache.seq_len.fill_(n)
            cache.ring_head.copy_(torch.as_tensor(rng.integers(0, p.ring_slots - p.sink if mask is None
                                                               else inputs.RECENT, size=B),
                                                  dtype=torch.int32))
            q = inputs.randn_bf16((B, 48, 128), seed * 100 + li + 50, "cuda")
            out = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((B, 48), dtype=torch.float32, device="cuda")
            self.layers.append((p, cache, q, out, lse))
            if product:
                max_ws = max(max_ws, duo.duo_decode_workspace_bytes(p, n))
        self.ws = torch.zeros((max_ws + 255) // 256 * 256, dtype=torch.uint8, device="cuda") if product else None
        self.launches_per_step = 2 * len(self.layers)
        self.unit = "GB/s"
        self.kernel = "40 x (decode_split + decode_merge), one CUDA graph"
        self.traffic_key = ("decode_split", "stack40")
        self.graph = None

    def eager_step(self, qs=None):
        for i, (p, cache, q, out, lse) in enumerate(self.layers):
            duo.duo_attn_decode(p, cache, q if qs is None else qs[i], self.w.seq_len, out, lse, self.ws)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.eager_step()          # warms up attribute setting outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.eager_step()
        torch.cuda.synchronize()

    def step(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()

    def e2e_buffers(self):
        self.h_q = [l[2].cpu().pin_memory() for l in self.layers]
        self.h_out = [torch.empty(l[3].shape, dtype=l[3].dtype).pin_memory() for l in self.layers]
        self.h_lse = [torch.empty(l[4].shape, dtype=l[4].dtype).pin_memory() for l in self.layers]
        self.d_q = [torch.empty_like(l[2]) for l in self.layers]
        h2d = sum(t.numel() * 2 for t in self.h_q)
        d2h = sum(t.numel() * 2 for t in self.h_out) + sum(t.numel() * 4 for t in self.h_lse)
        return h2d, d2h

    def e2e_step(self):
        for i in range(len(self.layers)):
            self.d_q[i].copy_(self.h_q[i], non_blocking=True)
        self.eager_step(self.d_q)
        for i, l in enumerate(self.layers):
            self.h_out[i].copy_(l[3], non_blocking=True)
            self.h_lse[i].copy_(l[4], non_blocking=True)

    def config(self):
        return {"workload": "stack40: one decode step through 40 layers (10 DuoAttention layers "
                            "3,7,...,39 with 2 of 8 heads full, 30 sliding-window layers of 512 "
                            "with sink logits), B=16, context 131072, CUDA graph",
                "batch_per_gpu": self.w.batch, "context": self.w.seq_len, "layers": 40,
                "l2": "inputs larger than L2 (22.6 GB of cache per step)"}

    def _host_layer(self, li, seqs):
        """The oracle's view of layer li restricted to the sequences seqs."""
        import oracle
        p, cache, q, _, _ = self.layers[li]
        b0, b1 = seqs
        ol = oracle.Layer(b1 - b0, 48, 8, 128, p.sink, p.recent, p.window, p.softmax_scale,
                          tuple(p.full_mask), None if p.sink_logit is None else p.sink_logit.cpu().numpy())
        hc = oracle.Cache(ol, cache.capacity if p.n_full else 1)
        if p.n_full:
            hc.full_k = inputs.bits(cache.full_k[b0:b1])
            hc.full_v = inputs.bits(cache.full_v[b0:b1])
        hc.strm_k = inputs.bits(cache.strm_k[b0:b1])
        hc.strm_v = inputs.bits(cache.strm_v[b0:b1])
        hc.seq_len = cache.seq_len[b0:b1].cpu().numpy().astype(np.int32)
        hc.ring_head = cache.ring_head[b0:b1].cpu().numpy().astype(np.int32)
        n = self.w.seq_len
        nbytes = decode_bytes(b1 - b0, n, p.n_full, p.n_ring, p.window if p.window else p.sink + p.recent)
        return ol, hc, inputs.bits(q[b0:b1]), nbytes

    def oracle_sample(self, budget_s: float = 15.0):
        """The oracle on two layers of the step: DuoAttention layer 3 for
        sequences 0-3 (48 full-head rows of 131072 keys per call, enough to keep
        the host threads busy) and sliding layer 0 for all 16 sequences."""
        import oracle
        units = [self._host_layer(3, (0, 4)), self._host_layer(0, (0, self.w.batch))]

        def run(u):
            oracle.attn_decode(u[0], u[1], u[2])

        done_bytes, t_total, used = timed_sample(units, run, lambda u: u[3], budget_s)
        threads = oracle.num_threads()
        return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": threads,
                "threads_busy": min(threads, 48), "kind": "oracle",
                "sample": f"{used} layer calls alternating DuoAttention layer 3 (sequences 0-3) and "
                          f"sliding layer 0 (all 16 sequences) of one step, float64, {t_total:.1f} s"}


class Prefill:
    """Prefill of one layer: prefill_16k (B=1, L=16384, 2 of 8 heads full) or
    sliding_32k (B=2, L=32768, window 512, sink logits, RMSNorm'd Q/K)."""

    def __init__(self, rank: int, name: str, product: bool = True):
        w = self.w = inputs.workload(name)
        B, L = w.batch, w.seq_len
        seed = rank_seed(w.seed, rank)
        sig = inputs.randn_f32((48,), seed + 9, "cuda") if w.sink_logit else None
        self.params = duo.DuoParams(B, 48, 8, 128, inputs.SINK, inputs.RECENT, w.window,
                                    128 ** -0.5, w.full_mask, sig)
        self.q = inputs.randn_bf16((B, L, 48, 128), seed, "cuda")
        self.k = inputs.randn_bf16((B, L, 8, 128), seed + 1, "cuda")
        self.v = inputs.randn_bf16((B, L, 8, 128), seed + 2, "cuda")
        if w.rmsnorm:
            self.q, self.k = inputs.rmsnorm_bf16(self.q), inputs.rmsnorm_bf16(self.k)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((B, 48, L), dtype=torch.float32, device="cuda")
        self.flops = prefill_flops(w)
        self.ws = torch.empty(duo.duo_prefill_workspace_bytes(), dtype=torch.uint8,
                              device="cuda") if product else None
        self.launches_per_step = 1      # prefill_fwd (plus a 4-byte memset of its work counter)
        self.unit = "TFLOP/s"
        self.kernel = "prefill_fwd"
        self.traffic_key = ("prefill_fwd", name)

    def step(self):
        duo.duo_attn_prefill(self.params, self.q, self.k, self.v, self.out, self.lse,
                             workspace=self.ws)

    def e2e_buffers(self):
        self.h_in = [t.cpu().pin_memory() for t in (self.q, self.k, self.v)]
        self.d_in = [torch.empty_like(t) for t in (self.q, self.k, self.v)]
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()
        return sum(t.numel() * 2 for t in self.h_in), self.h_out.numel() * 2 + self.h_lse.numel() * 4

    def e2e_step(self):
        for d, h in zip(self.d_in, self.h_in):
            d.copy_(h, non_blocking=True)
        duo.duo_attn_prefill(self.params, *self.d_in, self.out, self.lse, workspace=self.ws)
        self.h_out.copy_(self.out, non_blocking=True)
        self.h_lse.copy_(self.lse, non_blocking=True)

    def config(self):
        return {"workload": f"{self.w.name}: prefill B={self.w.batch}, L={self.w.seq_len}",
                "window": self.w.window, "full_mask": list(self.w.full_mask),
                "l2": "inputs larger than L2"}

    def oracle_sample(self, budget_s: float = 15.0):
        """The oracle on seeded sets of query positions of sequence 0 (every
        query head of each position in one call), cycled until the budget;
        TFLOP/s of the attended pairs those rows cover (4 * 128 flop each)."""
        import oracle
        w, p = self.w, self.params
        L = w.seq_len
        sig = None if p.sink_logit is None else p.sink_logit.cpu().numpy()
        ol = oracle.Layer(1, 48, 8, 128, p.sink, p.recent, p.window, p.softmax_scale,
                          tuple(p.full_mask), sig)
        qb, kb, vb = (inputs.bits(t[:1]) for t in (self.q, self.k, self.v))
        rng = np.random.default_rng(w.seed + 77)
        units = []
        for _ in range(64):
            pos = np.sort(rng.integers(0, L, size=16))
            rows = np.asarray([h * L + i for h in range(48) for i in pos], dtype=np.int64)
            pairs = 0
            for g in range(8):
                span = p.window if p.window else (None if p.full_mask[g] else p.sink + p.recent)
                per = [i + 1 if span is None else min(i + 1, span) for i in pos]
                pairs += 6 * int(sum(per))
            units.append((rows, pairs * 4 * 128))

        def run(u):
            oracle.attn_prefill(ol, qb, kb, vb, rows=u[0])

        done, t_total, used = timed_sample(units, run, lambda u: u[1], budget_s)
        return {"value": done / t_total / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                "kind": "oracle",
                "sample": f"{used} calls of 768 rows (16 seeded query positions of sequence 0 x 48 "
                          f"query heads), {done / 1e9:.1f} GFLOP of attended pairs, float64, "
                          f"{t_total:.1f} s"}


class VerifyB32(DecodeB32):
    """Verify-block decode on decode_b32's caches: a block of 8 query tokens per
    sequence (the DFlash verify shape) against 32768 cached tokens plus the
    block's own keys, cache untouched.  GB/s of the bytes it must read: the
    cached K/V rows the block's queries attend to (each read once for all 8
    queries), the block's K/V, q and out."""

    Q_LEN = 8
    oracle_sample = None

    def __init__(self, rank: int, product: bool = True):
        super().__init__(rank, product)
        B, n, k = self.w.batch, self.w.seq_len, self.Q_LEN
        seed = rank_seed(self.w.seed, rank)
        self.qb = inputs.randn_bf16((B, k, 48, 128), seed + 6, "cuda")
        self.kb = inputs.randn_bf16((B, k, 8, 128), seed + 7, "cuda")
        self.vb = inputs.randn_bf16((B, k, 8, 128), seed + 8, "cuda")
        self.outb = torch.empty_like(self.qb)
        self.lseb = torch.empty((B, k, 48), dtype=torch.float32, device="cuda")
        if product:
            nb = duo.duo_decode_block_workspace_bytes(self.params, k, n)
            self.wsb = torch.zeros((nb + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
        n_full, n_ring = self.params.n_full, self.params.n_ring
        self.bytes = verify_bytes(B, n, k, n_full, n_ring)
        self.kernel = "decode_block_split + decode_block_merge (one duo_attn_decode_block call)"
        self.traffic_key = ("decode_block_split", "verify_b32")

    def step(self):
        duo.duo_attn_decode_block(self.params, self.cache, self.qb, self.kb, self.vb, self.w.seq_len,
                                  self.outb, self.lseb, self.wsb)

    def e2e_buffers(self):
        self.h_in = [t.cpu().pin_memory() for t in (self.qb, self.kb, self.vb)]
        self.d_in = [torch.empty_like(t) for t in (self.qb, self.kb, self.vb)]
        self.h_out = torch.empty(self.outb.shape, dtype=self.outb.dtype).pin_memory()
        self.h_lse = torch.empty(self.lseb.shape, dtype=self.lseb.dtype).pin_memory()
        return sum(t.numel() * 2 for t in self.h_in), self.h_out.numel() * 2 + self.h_lse.numel() * 4

    def e2e_step(self):
        for d, h in zip(self.d_in, self.h_in):
            d.copy_(h, non_blocking=True)
        duo.duo_attn_decode_block(self.params, self.cache, *self.d_in, self.w.seq_len, self.outb,
                                  self.lseb, self.wsb)
        self.h_out.copy_(self.outb, non_blocking=True)
        self.h_lse.copy_(self.lseb, non_blocking=True)

    def config(self):
        return {"workload": "verify_b32: block of 8 query tokens, B=32, context 32768, "
                            "2 of 8 KV heads full"}


class ChunkPrefill:
    """Chunked prefill: a 4096-token prompt chunk that continues 28672 cached
    tokens (32768 in all), B=1, prefill_16k's head mask, through
    duo_attn_decode_block's long-block path (the cache untouched).  TFLOP/s of
    the attended (query, key) pairs, 4 * 128 flop each."""

    CACHED, CHUNK = 28672, 4096

    def __init__(self, rank: int, product: bool = True):
        w = self.w = inputs.workload("prefill_16k")
        B, n, C = 1, self.CACHED, self.CHUNK
        seed = rank_seed(w.seed + 31, rank)
        self.params = duo.DuoParams(B, 48, 8, 128, inputs.SINK, inputs.RECENT, 0, 128 ** -0.5,
                                    w.full_mask, None)
        self.cache = duo.DuoCache.allocate(self.params, n)
        for i, t in enumerate((self.cache.full_k, self.cache.full_v, self.cache.strm_k,
                               self.cache.strm_v)):
            inputs.randn_bf16_into(t, seed * 10 + i)
        self.cache.seq_len.fill_(n)
        self.cache.ring_head.fill_(int(np.random.default_rng(seed).integers(0, inputs.RECENT)))
        self.q = inputs.randn_bf16((B, C, 48, 128), seed + 5, "cuda")
        self.kb = inputs.randn_bf16((B, C, 8, 128), seed + 6, "cuda")
        self.vb = inputs.randn_bf16((B, C, 8, 128), seed + 7, "cuda")
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((B, C, 48), dtype=torch.float32, device="cuda")
        if product:
            nb = duo.duo_decode_block_workspace_bytes(self.params, C, n)
            self.ws = torch.empty((nb + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
        n_full = sum(1 for g in range(8) if w.full_mask[g])
        span = inputs.SINK + inputs.RECENT
        pairs = 6 * n_full * (C * n + C * (C + 1) // 2) + 6 * (8 - n_full) * C * span
        self.flops = 4 * 128 * pairs * B
        self.launches_per_step = 3      # prefill_fwd twice (cached keys, own keys) + block_combine
        self.unit = "TFLOP/s"
        self.kernel = "prefill_fwd (cache mode) + prefill_fwd + block_combine (one duo_attn_decode_block call)"
        self.traffic_key = ("prefill_fwd+block_combine", "chunk_32k")

    def step(self):
        duo.duo_attn_decode_block(self.params, self.cache, self.q, self.kb, self.vb, self.CACHED,
                                  self.out, self.lse, self.ws)

    def e2e_buffers(self):
        self.h_in = [t.cpu().pin_memory() for t in (self.q, self.kb, self.vb)]
        self.d_in = [torch.empty_like(t) for t in (self.q, self.kb, self.vb)]
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()
        return sum(t.numel() * 2 for t in self.h_in), self.h_out.numel() * 2 + self.h_lse.numel() * 4

    def e2e_step(self):
        for d, h in zip(self.d_in, self.h_in):
            d.copy_(h, non_blocking=True)
        duo.duo_attn_decode_block(self.params, self.cache, *self.d_in, self.CACHED, self.out, self.lse,
                                  self.ws)
        self.h_out.copy_(self.out, non_blocking=True)
        self.h_lse.copy_(self.lse, non_blocking=True)

    def config(self):
        return {"workload": f"chunk_32k: chunked prefill, B=1, a {self.CHUNK}-token chunk after "
                            f"{self.CACHED} cached tokens, 2 of 8 KV heads full",
                "full_mask": list(self.w.full_mask), "l2": "inputs larger than L2"}

    def oracle_sample(self, budget_s: float = 15.0):
        """The oracle's block decode on seeded sets of 16 chunk positions (every
        query head of each, in one call), cycled until the budget; TFLOP/s of the
        attended pairs those rows cover."""
        import oracle
        p, n, C = self.params, self.CACHED, self.CHUNK
        ol = oracle.Layer(1, 48, 8, 128, p.sink, p.recent, 0, p.softmax_scale, tuple(p.full_mask), None)
        hc = oracle.Cache(ol, n)
        hc.full_k[...] = inputs.bits(self.cache.full_k)
        hc.full_v[...] = inputs.bits(self.cache.full_v)
        hc.strm_k[...] = inputs.bits(self.cache.strm_k)
        hc.strm_v[...] = inputs.bits(self.cache.strm_v)
        hc.seq_len[...] = self.cache.seq_len.cpu().numpy()
        hc.ring_head[...] = self.cache.ring_head.cpu().numpy()
        qb, kb, vb = (inputs.bits(t) for t in (self.q, self.kb, self.vb))
        rng = np.random.default_rng(self.w.seed + 78)
        n_full = sum(1 for g in range(8) if p.full_mask[g])
        units = []
        for _ in range(64):
            pos = np.sort(rng.integers(0, C, size=16))
            rows = np.asarray([t * 48 + h for t in pos for h in range(48)], dtype=np.int64)
            pairs = sum(6 * n_full * (n + int(t) + 1) + 6 * (8 - n_full) * (p.sink + p.recent) for t in pos)
            units.append((rows, pairs * 4 * 128))

        def run(u):
            oracle.attn_decode_block(ol, hc, qb, kb, vb, rows=u[0])

        done, t_total, used = timed_sample(units, run, lambda u: u[1], budget_s)
        return {"value": done / t_total / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                "kind": "oracle",
                "sample": f"{used} calls of 768 rows (16 seeded chunk positions x 48 query heads), "
                          f"{done / 1e9:.1f} GFLOP of attended pairs, float64, {t_total:.1f} s"}


class Prep:
    """The fused query/key preparation + append of a 16384-token prompt on the
    prefill_16k layer (2 of 8 KV heads full): RMSNorm + YaRN RoPE of q and k in
    place, prepared k and v appended to the cache.  HBM-bound: GB/s of the
    bytes it must move (q and k read and written, the surviving K/V rows
    written, their v rows read)."""

    APPENDS = 64                      # capacity in prompts; the cache is reset when full

    def __init__(self, rank: int, product: bool = True):
        w = self.w = inputs.workload("prefill_16k")
        B, L = w.batch, w.seq_len
        seed = rank_seed(w.seed, rank)
        self.params = duo.DuoParams(B, 48, 8, 128, inputs.SINK, inputs.RECENT, 0, 128 ** -0.5,
                                    w.full_mask, None)
        self.cache = duo.DuoCache.allocate(self.params, L * self.APPENDS)
        self.q = inputs.randn_bf16((B, L, 48, 128), seed, "cuda")
        self.k = inputs.randn_bf16((B, L, 8, 128), seed + 1, "cuda")
        self.v = inputs.randn_bf16((B, L, 8, 128), seed + 2, "cuda")
        self.prep = duo.DuoQKPrep(
            q_norm_weight=(1 + 0.1 * inputs.randn_f32((128,), seed + 3)).to("cuda", torch.bfloat16),
            k_norm_weight=(1 + 0.1 * inputs.randn_f32((128,), seed + 4)).to("cuda", torch.bfloat16))
        self.appends = 0
        n_full, n_ring = self.params.n_full, self.params.n_ring
        kept = B * (n_full * L + n_ring * inputs.RECENT)   # rows each later append keeps
        self.bytes = 2 * (self.q.numel() + self.k.numel()) * 2 + 3 * kept * 256
        self.launches_per_step = 2      # qk_prep_append + kv_append_commit
        self.unit = "GB/s"
        self.kernel = "qk_prep_append"
        self.traffic_key = ("qk_prep_append", "prep_16k")

    def step(self):
        if self.appends == self.APPENDS:
            self.cache.seq_len.zero_()
            self.cache.ring_head.zero_()
            self.appends = 0
        duo.duo_kv_append_prep(self.params, self.cache, self.prep, self.q, self.k, self.v)
        self.appends += 1

    def config(self):
        return {"workload": "prep_16k: RMSNorm + YaRN RoPE of q/k in place + append, B=1, 16384 tokens"}


class DecodeSmall:
    """The single-layer workload end to end, B=1, full heads {0,3,5,6}: the
    1024-token prompt is prefilled and appended, then 16 decode steps each
    append one token and decode it.  Latency-bound, reported in microseconds:
    the prompt's prefill, and the decode steps.  The 16 steps (each an append
    and a decode, four kernels) are captured in one CUDA graph that first puts
    the cache state back to the end of the prompt; one replay is 16 steps.
    The caches (about 5 MB) would stay in L2, so L2 is flushed before every
    timed replay and every timed prefill (and only the call is timed)."""

    STEPS = 16

    def __init__(self, rank: int, product: bool = True):
        w = self.w = inputs.workload("decode_small")
        seed = rank_seed(w.seed, rank)
        self.params = duo.DuoParams(1, 48, 8, 128, inputs.SINK, inputs.RECENT, 0, 128 ** -0.5,
                                    w.full_mask, None)
        self.n0 = w.seq_len
        self.cap = w.seq_len + self.STEPS
        self.cache = duo.DuoCache.allocate(self.params, self.cap)
        self.qp = inputs.randn_bf16((1, w.seq_len, 48, 128), seed + 2, "cuda")
        self.kp = inputs.randn_bf16((1, w.seq_len, 8, 128), seed, "cuda")
        self.vp = inputs.randn_bf16((1, w.seq_len, 8, 128), seed + 1, "cuda")
        self.outp = torch.empty_like(self.qp)
        self.lsep = torch.empty((1, 48, w.seq_len), dtype=torch.float32, device="cuda")
        S = self.STEPS
        self.k1 = inputs.randn_bf16((S, 1, 1, 8, 128), seed + 3, "cuda")
        self.v1 = inputs.randn_bf16((S, 1, 1, 8, 128), seed + 4, "cuda")
        self.q1 = inputs.randn_bf16((S, 1, 48, 128), seed + 5, "cuda")
        self.out = torch.empty((S, 1, 48, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((S, 1, 48), dtype=torch.float32, device="cuda")
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")   # 2 x L2
        self.unit = "us/step"
        self.kernel = "kv_append_small + decode_split + decode_merge"
        self.launches_per_step = 3
        self.graph = None
        if product:
            self.ws_p = torch.empty(duo.duo_prefill_workspace_bytes(), dtype=torch.uint8, device="cuda")
            self.ws = duo.workspace_for(self.params, self.cap)
            self.prefill()
            duo.duo_kv_append(self.params, self.cache, self.kp, self.vp)
            self.seq0 = self.cache.seq_len.clone()
            self.ring0 = self.cache.ring_head.clone()

    def prefill(self):
        duo.duo_attn_prefill(self.params, self.qp, self.kp, self.vp, self.outp, self.lsep,
                             workspace=self.ws_p)

    def steps(self):
        """The cache back to the end of the prompt, then the 16 decode steps."""
        self.cache.seq_len.copy_(self.seq0)
        self.cache.ring_head.copy_(self.ring0)
        for s in range(self.STEPS):
            duo.duo_kv_append(self.params, self.cache, self.k1[s], self.v1[s])
            duo.duo_attn_decode(self.params, self.cache, self.q1[s], self.n0 + s + 1, self.out[s],
                                self.lse[s], self.ws)

    def capture(self):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.steps()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.steps()
        torch.cuda.synchronize()

    def replay(self):
        self.graph.replay()

    def timed_each(self, fn, reps):
        """Device time of reps calls of fn, L2 flushed before each: CUDA events
        around every call on the launching stream; returns the mean seconds."""
        stream = torch.cuda.current_stream()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize()
        for a, b in evs:
            self.flush.fill_(1)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / 1e3 / reps

    def oracle_sample(self, budget_s: float = 15.0):
        """The oracle on the same workload: the prompt's prefill (every row) and
        the 16 decode steps against its own sequentially appended cache, each
        timed on the host cores; repeated while the budget lasts."""
        import oracle
        p = self.params
        ol = oracle.Layer(1, 48, 8, 128, p.sink, p.recent, 0, p.softmax_scale, tuple(p.full_mask), None)
        qb, kb, vb = inputs.bits(self.qp), inputs.bits(self.kp), inputs.bits(self.vp)
        k1, v1, q1 = inputs.bits(self.k1), inputs.bits(self.v1), inputs.bits(self.q1)
        t_pre, t_dec, runs = 0.0, 0.0, 0
        while runs == 0 or t_pre + t_dec < budget_s:
            t0 = time.perf_counter()
            oracle.attn_prefill(ol, qb, kb, vb)
            t1 = time.perf_counter()
            hc = oracle.Cache(ol, self.cap)
            oracle.kv_append(ol, hc, kb, vb)
            t_dec_run = 0.0
            for s in range(self.STEPS):
                t2 = time.perf_counter()
                oracle.kv_append(ol, hc, k1[s], v1[s])
                oracle.attn_decode(ol, hc, q1[s])
                t_dec_run += time.perf_counter() - t2
            t_pre += t1 - t0
            t_dec += t_dec_run
            runs += 1
        return {"value": round(t_dec / (runs * self.STEPS) * 1e6, 2), "unit": "us/step",
                "prefill_us": round(t_pre / runs * 1e6, 2), "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"{runs} runs of the whole workload (prefill of the 1024-token prompt, every row, "
                          f"then 16 x (append + decode)), float64"}

    def measure_line(self, reps, warmup, cpu_budget=0.0):
        self.capture()
        for _ in range(warmup):
            self.replay()
            self.prefill()
        torch.cuda.synchronize()
        if duo.duo_get_device_status() != duo.DUO_OK:
            raise RuntimeError("device status set during warm-up")
        with ClockSampler(torch.cuda.current_device()) as clk:
            clk.begin()
            t_graph = self.timed_each(self.replay, reps)
            t_eager = self.timed_each(self.steps, reps)
            t_prefill = self.timed_each(self.prefill, reps)
            clk.end()
        if duo.duo_get_device_status() != duo.DUO_OK:
            raise RuntimeError("device status set during timing")
        S = self.STEPS
        return {"value": round(t_graph / S * 1e6, 2), "unit": "us/step", "higher_is_better": False,
                "steps": reps * S, "kernel": self.kernel,
                "prefill_us": round(t_prefill * 1e6, 2),
                "eager_us_per_step": round(t_eager / S * 1e6, 2),
                "gpu_launches": reps * (S * self.launches_per_step + 1),
                "note": "decode steps replayed from one CUDA graph of 16 steps (append + decode each); "
                        "prefill_us: the 1024-token prompt's duo_attn_prefill; L2 flushed before "
                        "every timed call",
                "clocks": clk.summary(),
                **({"cpu_baseline": self.oracle_sample(cpu_budget)} if cpu_budget > 0 else {})}

    def config(self):
        return {"workload": "decode_small: B=1, prefill of a 1024-token prompt, then 16 x "
                            "(append one token + decode)"}


WORKLOADS = {"decode_b32": DecodeB32, "stack40": Stack40, "decode_small": DecodeSmall, "prep_16k": Prep,
             "verify_b32": VerifyB32,
             "prefill_16k": lambda rank, product=True: Prefill(rank, "prefill_16k", product),
             "sliding_32k": lambda rank, product=True: Prefill(rank, "sliding_32k", product),
             "chunk_32k": ChunkPrefill}
SECONDARY = ("stack40", "verify_b32", "prefill_16k", "sliding_32k", "prep_16k", "decode_small", "chunk_32k")


# ------------------------------------------------------------------ timing
PREROLL_CYCLES = 2_000_000     # ~1 ms device spin queued ahead of the start event


def time_steps(fn, steps, stream, world, clocks=None):
    """Device time of `steps` calls of fn: CUDA events on the launching stream,
    barrier + synchronize on both sides.  A ~1 ms spin kernel is queued before
    the start event, so the host's time to issue the first step's launches is
    not counted as idle device time inside the region (every step's device
    work still is)."""
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(PREROLL_CYCLES)
    start.record(stream)
    if clocks is not None:
        clocks.begin()
    for _ in range(steps):
        fn()
    stop.record(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.end()
    barrier(world)
    return start.elapsed_time(stop) / 1e3


def measure(wl, steps, warmup, world):
    """Warm-up, then `steps` timed steps (CUDA events on the launching stream,
    barrier + synchronize on both sides); returns (seconds per step of the
    slowest rank, clock summary)."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    status = duo.duo_get_device_status()
    if status != duo.DUO_OK:
        raise RuntimeError(f"device status {status} during warm-up")
    with ClockSampler(torch.cuda.current_device()) as clk:
        t = time_steps(wl.step, steps, stream, world, clk)
    t = max_over_ranks(t, world)
    status = duo.duo_get_device_status()
    if status != duo.DUO_OK:
        raise RuntimeError(f"device status {status} during timing")
    return t / steps, clk.summary()


CSRC = os.path.join(ROOT, "kv_cache_reduction_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")


KERNEL_SOURCES = {"decode_split": ("decode.cuh", "ptx.cuh", "kv_append.cuh"),
                  "prefill_fwd": ("prefill.cuh", "ptx.cuh"),
                  "decode_block_split": ("decode_block.cuh", "decode.cuh", "ptx.cuh", "kv_append.cuh"),
                  "qk_prep_append": ("qk_prep.cuh", "kv_append.cuh", "ptx.cuh"),
                  # the chunked-prefill step: both prefill_fwd passes and block_combine
                  "prefill_fwd+block_combine": ("prefill.cuh", "decode_block.cuh", "ptx.cuh")}


def sources_digest(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture, or None once the
    kernel's sources differ from the ones that were profiled."""
    digest = sources_digest(kernel)
    try:
        with open(TRAFFIC_FILE) as fh:
            for line in fh:
                if line.startswith("#") or not line.strip():
                    continue
                kv = dict(tok.split("=", 1) for tok in line.split())
                if kv.get("kernel") == kernel and kv.get("workload") == workload and \
                        kv.get("sources") == digest:
                    return int(kv["dram_bytes_per_launch"])
    except OSError:
        pass
    return None


def roofline(wl, per_step, pk, pk_kind):
    if wl.unit == "GB/s":
        achieved = wl.bytes / per_step / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": None,
                "peak_source": f"{pk_kind} hbm_gbs (copy bandwidth)"}
    achieved = wl.flops / per_step / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4), "traffic": None,
            "peak_source": f"{pk_kind} bf16_tflops (burst cuBLAS GEMM)"}


def units(wl):
    return wl.bytes / 1e9 if wl.unit == "GB/s" else wl.flops / 1e12


def measure_line(wl, args, world, rank, steps, cpu_budget, pk, pk_kind):
    """One workload's line: device-timed value and roofline, the clocks, the
    end-to-end figure through the binding with host buffers, and (rank 0 of a
    one-GPU run) the oracle on the host cores."""
    per_step, clocks = measure(wl, steps, args.warmup, world)
    value = aggregate(units(wl), world, per_step)
    rf = roofline(wl, per_step, pk, pk_kind)
    rf["kernel"] = wl.kernel
    key = getattr(wl, "traffic_key", None)
    if key is not None:
        rf["traffic"] = measured_traffic(*key)
        rf["traffic_unit"] = "bytes per step (ncu dram read + write of the kernel's launches)"
    res = {"value": round(value, 2), "unit": wl.unit, "ms_per_step": round(per_step * 1e3, 4),
           "steps": steps, "roofline": rf, "gpu_launches": wl.launches_per_step * steps,
           "clocks": clocks}
    if getattr(wl, "e2e_step", None) is not None:
        h2d, d2h = wl.e2e_buffers()
        for _ in range(args.warmup):
            wl.e2e_step()
        torch.cuda.synchronize()
        t_e2e = max_over_ranks(time_steps(wl.e2e_step, steps, torch.cuda.current_stream(), world),
                               world) / steps
        res["e2e"] = {"value": round(aggregate(units(wl), world, t_e2e), 2), "unit": wl.unit,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": round(t_e2e * 1e3, 4),
                      "path": "pinned host inputs -> device, the library call, outputs -> pinned host"}
    if rank == 0 and world == 1 and cpu_budget > 0 and getattr(wl, "oracle_sample", None) is not None:
        res["cpu_baseline"] = wl.oracle_sample(cpu_budget)
    return res


def run_ours(args, world, rank):
    pk, pk_kind = peaks()
    wl = WORKLOADS[args.workload](rank)
    budget = 0.0 if args.no_cpu_baseline else args.cpu_budget
    line = measure_line(wl, args, world, rank, args.steps, budget, pk, pk_kind)
    res = {"metric": METRIC, "value": line["value"], "unit": wl.unit, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": line["ms_per_step"],
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded N(0,1) bf16 inputs and caches)",
           "config": {**wl.config(), "parallelism": f"dp{world} (independent batches, no collective)"},
           "roofline": line["roofline"], "gpu_launches": line["gpu_launches"], "clocks": line["clocks"]}
    for k in ("e2e", "cpu_baseline"):
        if k in line:
            res[k] = line[k]
    if "cpu_baseline" in res:
        # the same oracle on one host thread, on a shorter bounded sample
        import oracle
        n_threads = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            one = wl.oracle_sample(max(1.0, args.cpu_budget / 3))
        finally:
            oracle.set_num_threads(n_threads)
        res["cpu_baseline"]["single_thread"] = {"value": one["value"], "unit": one["unit"],
                                                "cores": 1, "sample": one["sample"]}
    # the other workloads of the path, on this GPU, as context for the main line
    if args.secondary and args.workload == "decode_b32":
        del wl
        torch.cuda.empty_cache()
        sec = {}
        for name in SECONDARY:
            st = max(3, min(args.steps, 10))
            try:
                w2 = WORKLOADS[name](rank)
                if hasattr(w2, "measure_line"):
                    sec[name] = w2.measure_line(st, args.warmup, budget / 2 if world == 1 and rank == 0 else 0.0)
                else:
                    line = measure_line(w2, args, world, rank, st, budget / 2, pk, pk_kind)
                    line["frac"] = line["roofline"]["frac"]
                    line["bound"] = line["roofline"]["bound"]
                    line["kernel"] = w2.kernel
                    sec[name] = line
            except Exception as e:              # a secondary line must not lose the main one
                sec[name] = {"error": f"{type(e).__name__}: {e}"}
            w2 = None
            torch.cuda.empty_cache()
        res["secondary"] = sec
    return res


def run_reference(args, world, rank):
    """The float64 CPU oracle on this host's cores, on bounded samples of the
    workload; its inputs are built with torch alone (the library is not loaded)."""
    if rank != 0:
        return None
    if args.workload in ("verify_b32", "prep_16k", "chunk_32k"):
        return {"impl": "reference", "unavailable": f"no CPU oracle leg for {args.workload}; the "
                                                    "reference arm covers the workloads of the main line"}
    import oracle
    wl = WORKLOADS[args.workload](0, product=False)
    vals = []
    samples = []
    per = max(1.0, args.cpu_budget / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        r = wl.oracle_sample(per)
        if i >= args.warmup:
            vals.append(r["value"])
            samples.append(r["sample"])
    v = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": wl.unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16 caches and queries)",
            "config": {**wl.config(), "parallelism": "CPU oracle, rank 0 only"},
            "cpu_baseline": {"value": round(v, 4), "unit": wl.unit, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": samples[0]},
            "e2e": {"value": round(v, 4), "unit": wl.unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(k for k in WORKLOADS if k != "decode_small"),
                    default="decode_b32")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--secondary", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the 40-layer stack and the two prefill workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 only; no process group is needed
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        res = run_reference(args, world, rank)
        print(json.dumps(res), flush=True)
        return
    world, rank = dist_init()
    try:
        res = run_ours(args, world, rank) if args.impl == "ours" else run_reference(args, world, rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
