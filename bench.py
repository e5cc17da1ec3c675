"""Benchmark of the attention forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one call of the library's attention forward over one batch of the
workload (headline ``gqa_causal_prefill``: B 4, 32 query / 8 kv heads, L 4096,
D 128, bf16, causal).  Inputs are synthetic (seeded N(0,1)), resident in HBM
before the timed region; their footprint (335 MB) is larger than L2, so no
flush is needed between steps.  Timing: W untimed steps, then blocks of
exactly K steps, each bracketed by a barrier + synchronize and timed by CUDA
events on the launching stream, repeated until at least --min-timed-s seconds
(default 1) have been timed; ms_per_step is the median block's, max over
ranks; the SM clock is sampled over all blocks.  The metric is FLOP/s with
causal-adjusted (kept-pair) FLOPs: sum over (b, h) of 2 * (Dqk + Dv) * kept
pairs.

On one GPU the same line also carries, under ``workloads``, the other bf16
configurations timed the same way: ``mla_varlen_prefill`` (packed MLA, 8
sequences), ``blockkv_rolling`` (one step is the whole 16-chunk rolling-cache
loop through the fused chunk call, timed as a CUDA graph of that loop, plus the
same loop through the separate calls with their phase times) and
``long_gqa_causal`` (L 65536); the keep-mask throughput at the GQA shapes; and
the latency of the page example (fp32, no mask / keep-mask / additive mask).

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of the
headline workload (independent batches: weak scaling, no collective on the
data path); `value` = all ranks' FLOPs / the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only), the slow baseline arm.

``--workload NAME`` makes NAME the headline (with ``--no-extras``: only NAME,
for profilers).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_forward_tmem_b200 import parallel  # noqa: E402
from attention_forward_tmem_b200 import workloads as W  # noqa: E402

METRIC = "attention fwd TFLOP/s (causal-adjusted) and % of B200 dense BF16 tensor peak"
DATASHEET_BF16_TFLOPS = 2250.0        # NVIDIA B200 dense BF16, for the second peak reading
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# sources of the timed kernel (bf16: the two-tile kernel); a committed ncu
# traffic figure is only reported while these are unchanged
KERNEL_SOURCES = ["attention_forward_tmem_b200/csrc/attn_pingpong.cuh",
                  "attention_forward_tmem_b200/csrc/attn_common.cuh",
                  "attention_forward_tmem_b200/csrc/sm100_ptx.cuh",
                  "attention_forward_tmem_b200/csrc/attn_params.h"]


# ----------------------------------------------------------------- helpers

def measured_peaks():
    """Peak denominators: the generated MEASURED_PEAKS.json when present
    (its bf16 sustained figure under whichever key holds it), else the
    fallback figures of this GPU pool."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        out = dict(d)
        if "bf16_tflops_sustained" not in out:
            cand = [v for k, v in d.items() if "sustained" in k and "bf16" in k and isinstance(v, (int, float))]
            out["bf16_tflops_sustained"] = cand[0] if cand else out["bf16_tflops"]
        return out, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", f"attn_fwd_{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    mh = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", txt)
    mt = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not mh or not mt or mh.group(1) != kernel_hash():
        return None
    return float(mt.group(1))


def kept_pairs_causal(lq, lk):
    """Kept (query, key) pairs of one head under the bottom-right causal mask."""
    off = lk - lq
    total = 0
    for i in range(lq):
        total += max(0, min(lk, i + off + 1))
    return total


class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons) every 10 ms on a thread."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - NVML missing
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.01)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------- workloads

def config_of(name):
    """The `config` object of the JSON line (both arms)."""
    w = W.WORKLOADS[name]
    if name == "mla_varlen_prefill":
        lens = W.seqlens(w.batch, 512, 4096, W.SEED).tolist()
        return {"workload": name, "batch": w.batch, "seqlens": lens, "n_tokens": int(sum(lens)),
                "head_num": w.head_num, "head_dim": w.dqk, "rope_dim": w.drope, "mask": "causal"}
    if name == "blockkv_rolling":
        c = W.BLOCKKV
        return {"workload": name, "batch": 1, "head_num": w.head_num, "head_dim": w.dqk,
                "chunk_size": c["chunk_size"], "sink_size": c["sink_size"],
                "window_size": c["window_size"], "n_chunks": c["n_chunks"], "mask": "none",
                "step": "16 chunks: cache write + attention over the visible keys"}
    return {"workload": name, "batch": w.batch, "head_num": w.head_num,
            "kv_head_num": w.kv_head_num, "seq_len": w.seq, "head_dim": w.dqk, "mask": w.mask}


class Workload:
    """One step's inputs and the call that runs it through the public API."""

    def __init__(self, name, device, seq_len=None):
        from attention_forward_tmem_b200 import api
        self.api = api
        self.name = name
        self.device = device
        w = W.WORKLOADS[name]
        if seq_len and name in ("gqa_causal_prefill", "long_gqa_causal"):
            w = dataclasses.replace(w, seq=seq_len)      # a shorter case of the same shape (profiling)
        self.w = w
        self.launches_per_step = 1
        if name in ("gqa_causal_prefill", "long_gqa_causal"):
            q, k, v = W.dense_inputs(w.batch, w.head_num, w.kv_head_num, w.seq, w.seq, w.dqk, w.dv,
                                     w.dtype, W.SEED, w.input_scale)
            self.host = {"q": q, "k": k, "v": v}
            self.flops = w.batch * w.head_num * 2 * (w.dqk + w.dv) * kept_pairs_causal(w.seq, w.seq)
        elif name == "mla_varlen_prefill":
            d = W.mla_varlen_prefill()
            self.host = d
            lens = d["q_seqlen"].tolist()
            self.flops = sum(w.head_num * 2 * (w.dqk + w.drope + w.dv) * kept_pairs_causal(L, L)
                             for L in lens)
            self.launches_per_step = 2          # schedule + attention
        else:
            raise SystemExit(f"bench workload {name!r} is not a single-call workload")
        self.config = config_of(name)
        if "seq_len" in self.config:
            self.config["seq_len"] = w.seq
        self.out_host = None

    def to_device(self):
        self.dev = {k: v.to(self.device) for k, v in self.host.items()}
        self.out = self._alloc_out()

    def _alloc_out(self):
        q = self.dev["q"]
        if self.name == "mla_varlen_prefill":
            return torch.empty(q.shape[0], q.shape[1], self.w.dv, dtype=q.dtype, device=self.device)
        return torch.empty(q.shape[:3] + (self.w.dv,), dtype=q.dtype, device=self.device)

    def step(self, dev=None, out=None):
        d = dev or self.dev
        kw = dict(mask_type=self.api.MaskType.CAUSAL, qk_scale=self.w.qk_scale,
                  out=self.out if out is None else out)
        if self.name == "mla_varlen_prefill":
            kw.update(qrope=d["qrope"], krope=d["krope"], q_seqlen=d["q_seqlen"],
                      kv_seqlen=d["kv_seqlen"])
        self.api.attn_fwd(d["q"], d["k"], d["v"], **kw)

    def host_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host.values())


class RollingWorkload:
    """The rolling BlockKVCache loop: one step = 16 chunks, each
    before_update -> update (cache write) -> cached views -> attention of the
    chunk's 1024 queries over the visible keys (no mask) -> after_update.
    The cache (sink 1024 + window 7168 positions) is re-created (host state
    only) at the start of every step, over the same device buffers."""

    def __init__(self, name, device):
        from attention_forward_tmem_b200 import api
        self.api = api
        self.name = name
        self.device = device
        self.w = w = W.WORKLOADS[name]
        c = W.BLOCKKV
        self.chunk, self.n_chunks = c["chunk_size"], c["n_chunks"]
        self.sink, self.window = c["sink_size"], c["window_size"]
        self.cache_len = self.sink + self.window
        self.host = {}
        for i in range(self.n_chunks):
            q, k, v = W.blockkv_chunk(i, w.head_num, self.chunk, w.dqk, w.dtype)
            self.host[f"q{i}"], self.host[f"k{i}"], self.host[f"v{i}"] = q, k, v
        self.vis = [min((i + 1) * self.chunk, self.cache_len) for i in range(self.n_chunks)]
        self.flops = sum(w.head_num * 2 * (w.dqk + w.dv) * self.chunk * n for n in self.vis)
        self.cache_bytes = self.n_chunks * 2 * 2 * w.head_num * self.chunk * w.dqk * 2  # k+v, read+write
        self.config = config_of(name)

    def launches_per_chunk(self, i):
        """Kernels one chunk launches: the attention kernel (which also writes
        the chunk into the cache), and the merge pass when the library splits
        the keys (dense layout, units < SMs)."""
        sm = torch.cuda.get_device_properties(self.device).multi_processor_count
        units = self.w.head_num * ((self.chunk + 255) // 256)
        n = 1
        if units < sm:
            n = max(1, min(sm // units, ((self.vis[i] + 127) // 128) // 4))
        return 1 + (1 if n > 1 else 0)

    @property
    def launches_per_step(self):
        return sum(self.launches_per_chunk(i) for i in range(self.n_chunks))

    def to_device(self):
        self.dev = {k: v.to(self.device) for k, v in self.host.items()}
        shape = (1, self.w.head_num, self.cache_len, self.w.dqk)
        self.kb = torch.zeros(shape, dtype=self.w.dtype, device=self.device)
        self.vb = torch.zeros(shape, dtype=self.w.dtype, device=self.device)
        self.out = torch.empty((self.n_chunks, 1, self.w.head_num, self.chunk, self.w.dv),
                               dtype=self.w.dtype, device=self.device)

    def step(self, dev=None, out=None):
        """The chunk loop through the fused call (cache write + attention in
        one kernel per chunk)."""
        d = dev or self.dev
        out = self.out if out is None else out
        cache = self.api.BlockKVCache(self.kb, self.vb, chunk_size=self.chunk, window_size=self.window,
                                      sink_size=self.sink)
        for i in range(self.n_chunks):
            cache.before_update(i)
            cache.update_attend(d[f"k{i}"], d[f"v{i}"], d[f"q{i}"], qk_scale=self.w.qk_scale, out=out[i])
            cache.after_update(i)

    def step_unfused(self, dev=None, out=None, events=None):
        """The same loop as separate calls: update (copy kernels), cached
        views, attention."""
        d = dev or self.dev
        out = self.out if out is None else out
        api = self.api
        cache = api.BlockKVCache(self.kb, self.vb, chunk_size=self.chunk, window_size=self.window,
                                 sink_size=self.sink)
        for i in range(self.n_chunks):
            if events is not None:
                torch.cuda._sleep(2_000_000)       # let the host queue the chunk's work
                events[i][0].record()
            cache.before_update(i)
            cache.update(d[f"k{i}"], d[f"v{i}"])
            if events is not None:
                events[i][1].record()
            api.attn_fwd(d[f"q{i}"], cache.cached_k(), cache.cached_v(), mask_type=api.MaskType.NONE,
                         qk_scale=self.w.qk_scale, out=out[i])
            if events is not None:
                events[i][2].record()
            cache.after_update(i)

    def host_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host.values())

    def phase_times(self):
        """(cache-write ms, attention ms) of one step, from events around each
        chunk's two phases (the host is kept ahead of the GPU)."""
        self.step_unfused()         # this stream's library workspace reaches its size
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(self.n_chunks)]
        self.step_unfused(events=ev)
        torch.cuda.synchronize()
        write = sum(e[0].elapsed_time(e[1]) for e in ev)
        attn = sum(e[1].elapsed_time(e[2]) for e in ev)
        return write, attn


class BlockTimer:
    """Times blocks of exactly `steps` steps with CUDA events on the launching
    stream (barrier + synchronize on both sides of every block), repeated
    until at least `min_s` seconds have been timed; the SM clock is sampled
    over all blocks.  ms_per_step is the median block's."""

    def __init__(self, steps, warmup, min_s, dist_on):
        self.steps, self.warmup, self.min_s, self.dist_on = steps, warmup, min_s, dist_on

    def run(self, enqueue_step, graph=False):
        stream = torch.cuda.current_stream()
        step_fn = enqueue_step
        g = None
        if graph:
            # the step captured once in a CUDA graph (after eager warm-up on the
            # capture stream, so that nothing is allocated during capture): times
            # the device work of a step made of many small calls
            s = torch.cuda.Stream()
            s.wait_stream(stream)
            with torch.cuda.stream(s):
                for _ in range(self.warmup):
                    enqueue_step()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                enqueue_step()
            torch.cuda.synchronize()
            step_fn = g.replay
        for _ in range(self.warmup):
            step_fn()
        torch.cuda.synchronize()
        blocks = []
        n_blocks = 1
        with ClockSampler(torch.cuda.current_device()) as clk:
            while len(blocks) < n_blocks:
                if self.dist_on:
                    torch.distributed.barrier()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(self.steps):
                    step_fn()
                e1.record(stream)
                torch.cuda.synchronize()
                blocks.append(e0.elapsed_time(e1))
                if len(blocks) == 1:
                    # every rank runs the same number of blocks
                    n = max(1, math.ceil(1e3 * self.min_s / max(blocks[0], 1e-3)))
                    if self.dist_on:
                        n = int(parallel.max_over_ranks(float(n), torch.device("cuda", torch.cuda.current_device())))
                    n_blocks = n
        del g
        return statistics.median(blocks) / self.steps, len(blocks), sum(blocks), clk.summary()


def time_e2e(wl, steps, warmup):
    """Same steps through the public API with host inputs: every step copies
    its q/k/v (+lengths) from pinned host memory to the device and reads its
    output back, all inside the timed region.  As a server streaming requests
    would, step i+1's uploads run on a second stream while step i computes and
    its output is read back (device inputs and outputs double-buffered; events
    order the buffer reuse), so the two copy directions and the compute
    overlap."""
    pinned = {k: v.pin_memory() for k, v in wl.host.items()}
    out_host = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
    dev = [{k: torch.empty_like(v, device=wl.device) for k, v in pinned.items()} for _ in range(2)]
    outs = [torch.empty_like(wl.out) for _ in range(2)]
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    loaded = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]

    def upload(i):
        b = i % 2
        copy.wait_event(freed[b])          # step i-2 has finished reading these buffers
        with torch.cuda.stream(copy):
            for k in pinned:
                dev[b][k].copy_(pinned[k], non_blocking=True)
            loaded[b].record(copy)

    def compute(i):
        b = i % 2
        comp.wait_event(loaded[b])
        wl.step(dev=dev[b], out=outs[b])
        freed[b].record(comp)
        out_host.copy_(outs[b], non_blocking=True)

    def run(n, start):
        copy.wait_event(start)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)

    e_w = torch.cuda.Event()
    e_w.record(comp)
    run(warmup, e_w)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(steps, e0)
    e1.record(comp)
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = out_host.numel() * out_host.element_size()
    return e0.elapsed_time(e1), h2d, d2h


# -------------------------------------------------------------- CPU oracle

def _oracle_rows_dense(w, rng, seed):
    """Rows of one GQA group of a dense causal workload, each over its full
    causal key range."""
    import oracle
    g = w.head_num // w.kv_head_num
    q, k, v = W.dense_inputs(1, g, 1, w.seq, w.seq, w.dqk, w.dv, w.dtype, seed, w.input_scale)

    def make(n):
        rows = np.stack([np.zeros(n, np.int64), rng.integers(0, g, n), rng.integers(0, w.seq, n)], 1)
        fl = float(sum(2 * (w.dqk + w.dv) * (int(r) + 1) for r in rows[:, 2]))
        return fl, lambda: oracle.sdpa_rows(q, k, v, rows, mask_kind="causal", qk_scale=w.qk_scale,
                                            head_num=g, kv_head_num=1)
    desc = f"one GQA group, rows uniform in [0, {w.seq}), each over its full causal key range"
    return make, 2 * (w.dqk + w.dv) * w.seq / 2, desc


def _oracle_rows_packed(w, rng, seed):
    """Rows of the packed MLA workload (its sequence lengths; one head, as every
    head costs the same per row), token-uniform, each over its causal range."""
    import oracle
    lens = W.seqlens(w.batch, 512, 4096, seed)
    d = W.packed_inputs(lens, lens, 1, 1, w.dqk, w.dv, w.drope, w.dtype, seed)
    L = lens.numpy().astype(np.int64)
    p = L / L.sum()

    def make(n):
        b = rng.choice(len(L), size=n, p=p)
        i = (rng.random(n) * L[b]).astype(np.int64)
        rows = np.stack([b, np.zeros(n, np.int64), i], 1)
        fl = float(np.sum(2 * (w.dqk + w.drope + w.dv) * (i + 1)))
        return fl, lambda: oracle.sdpa_rows(d["q"], d["k"], d["v"], rows, qrope=d["qrope"],
                                            krope=d["krope"], q_seqlen=lens, kv_seqlen=lens,
                                            mask_kind="causal", qk_scale=w.qk_scale)
    desc = "packed MLA sequences (one head), rows token-uniform, each over its causal key range"
    return make, 2 * (w.dqk + w.drope + w.dv) * float(np.sum(L * L) / np.sum(L)) / 2, desc


def _oracle_rows_rolling(w, rng, seed):
    """Rows of the rolling-cache loop (head 0; every head costs the same per
    row): chunk uniform, each row over the keys visible at that chunk (logical
    order; attention is order-free)."""
    import oracle
    from oracle.kvcache_model import BlockKVCacheModel
    c = W.BLOCKKV
    chunks = [tuple(t[:, :1] for t in W.blockkv_chunk(i, w.head_num, c["chunk_size"], w.dqk, w.dtype))
              for i in range(c["n_chunks"])]
    model = BlockKVCacheModel(c["sink_size"] + c["window_size"], c["chunk_size"], c["window_size"],
                              c["sink_size"])
    vis_ids = [model.logical_chunks(i) for i in range(c["n_chunks"])]

    def make(n):
        ci = rng.integers(0, c["n_chunks"], n)
        calls, fl = [], 0.0
        for i in sorted(set(ci.tolist())):
            m = int(np.sum(ci == i))
            rows = np.stack([np.zeros(m, np.int64), np.zeros(m, np.int64),
                             rng.integers(0, c["chunk_size"], m)], 1)
            kk = torch.cat([chunks[j][1] for j in vis_ids[i]], dim=2)
            vv = torch.cat([chunks[j][2] for j in vis_ids[i]], dim=2)
            fl += m * 2 * (w.dqk + w.dv) * kk.shape[2]
            calls.append((chunks[i][0], kk, vv, rows))

        def run():
            for q, kk, vv, rows in calls:
                oracle.sdpa_rows(q, kk, vv, rows, qk_scale=w.qk_scale)
        return fl, run
    desc = "rolling-cache rows of head 0, chunk uniform, each over the keys visible at its chunk"
    mean_vis = np.mean([len(v) * c["chunk_size"] for v in vis_ids])
    return make, 2 * (w.dqk + w.dv) * mean_vis, desc


def oracle_sample(name, budget_s=12.0, seed=7, n=None):
    """Time the fp64 oracle on rows of the workload (each over its full key
    range) for about `budget_s` seconds, or on `n` rows when given (no
    calibration).  Returns (TFLOP/s, threads, note, rows)."""
    import oracle
    w = W.WORKLOADS[name]
    rng = np.random.default_rng(seed)
    maker = {"mla_varlen_prefill": _oracle_rows_packed,
             "blockkv_rolling": _oracle_rows_rolling}.get(name, _oracle_rows_dense)
    make, per_row, desc = maker(w, rng, seed)

    def run(n):
        fl, fn = make(n)
        t0 = time.perf_counter()
        fn()
        return fl, time.perf_counter() - t0

    # Calibrate until a run takes a quarter of the budget (small runs are
    # dominated by per-call overhead and overstate the cost of a row), then
    # size the timed sample from that rate.
    n_max = 400000
    if n is not None:
        fl, dt = run(n)
    else:
        n = 64
        while True:
            fl, dt = run(n)
            if dt >= 0.25 * budget_s or n >= n_max:
                break
            n = int(min(n_max, max(2 * n, fl / max(dt, 1e-6) * budget_s * 0.3 / per_row)))
        n_final = int(min(n_max, max(n, fl / max(dt, 1e-6) * budget_s / per_row)))
        if n_final != n:
            n = n_final
            fl, dt = run(n)
    note = f"{n} query rows of {name} ({desc}), fp64 oracle, {dt:.1f} s"
    return fl / dt / 1e12, oracle.oracle_threads(), note, n


# -------------------------------------------------------------------- main

def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
        return True, torch.distributed.get_rank(), ws
    if args.gpus > 1:
        raise SystemExit("--gpus > 1 needs torchrun (one process per GPU)")
    return False, 0, 1


def reference_arm(args, rank, world):
    if rank != 0:
        return
    name = args.workload
    # Each step is a bounded sample sized so that warm-up plus timed steps
    # take about --ref-total-s seconds (at most 3 s a step): the row count is
    # calibrated on the first warm-up step and kept, with fresh rows per step.
    n_total = args.warmup + args.steps
    step_s = args.ref_step_s if args.ref_step_s > 0 else min(3.0, max(0.05, args.ref_total_s / n_total))
    per_step = []
    note = threads = rows = None
    for i in range(n_total):
        v, threads, note, rows = oracle_sample(name, budget_s=step_s, seed=100 + i, n=rows)
        if i >= args.warmup:
            per_step.append(v)
    val = statistics.mean(per_step)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_of(name), parallelism="host cores"),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": note},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def make_workload(name, device, seq_len=None):
    return RollingWorkload(name, device) if name == "blockkv_rolling" else Workload(name, device, seq_len)


def measure(wl, timer, args):
    """Device time of the workload's step (inputs resident); returns the
    workload's entry of the JSON line."""
    rolling = wl.name == "blockkv_rolling"
    extra = {}
    if rolling:
        try:
            ms, blocks, total, clocks = timer.run(wl.step, graph=True)
            how = "step = CUDA graph of the 16-chunk loop (the kernels the API launches)"
            ms_unf = None
            if not args.no_extras:
                ms_unf = timer.run(wl.step_unfused, graph=True)[0]
        except RuntimeError as e:          # capture refused: time the eager loop instead
            print(f"graph capture failed ({e}); timing the eager loop", file=sys.stderr)
            ms, blocks, total, clocks = timer.run(wl.step)
            ms_unf = None
            how = "step = eager 16-chunk loop (graph capture failed)"
        write_ms, attn_ms = (float("nan"), float("nan")) if args.no_extras else wl.phase_times()
        extra = {"fused_cache_write": True,
                 "unfused_ms_per_step": ms_unf,
                 "unfused_attention_ms_per_step": attn_ms, "unfused_cache_write_ms_per_step": write_ms,
                 "unfused_cache_write_gbs": wl.cache_bytes / (write_ms / 1e3) / 1e9,
                 "timing": how + "; unfused phase times from per-chunk events"}
    else:
        ms, blocks, total, clocks = timer.run(wl.step)
    wl.api.device_status()
    return ms, blocks, total, clocks, extra


def roofline_of(wl, ms, peaks, peak_kind):
    """The attention kernel's own rate (per launch, or for the rolling cache per
    step of fused attention + cache-write kernels and their merge passes)
    against the dense bf16 peak.  The timed region is a loop of at least a
    second, which runs under the 1 kW power cap, so the denominator is the
    sustained GEMM figure; the burst one is given beside it."""
    achieved = wl.flops / (ms / 1e3) / 1e12
    sustained, burst = peaks["bf16_tflops_sustained"], peaks["bf16_tflops"]
    return {"bound": "tensor", "achieved": achieved, "peak": sustained,
            "unit": "TFLOP/s", "frac": achieved / sustained,
            "frac_of_burst_peak": achieved / burst, "burst_peak": burst,
            "traffic": profiled_traffic(wl.name),
            "peak_source": (f"{peak_kind} bf16 sustained (MEASURED_PEAKS.json; seconds-long loop under "
                            "the power cap, as this timed region is)")
            if peak_kind == "measured" else "fallback 1.4 PFLOP/s sustained (1.59 burst)",
            "kernel": "wf::attn_fwd_pp_kernel" if wl.w.dtype == torch.bfloat16 else "wf::attn_fwd_kernel",
            "algorithmic_flops_per_launch": wl.flops}


def page_example_latency(device, calls=200):
    """Latency of the page example (fp32, q [2,8,32,64], k [2,8,48,64],
    v [2,8,48,96]) without a mask, with its keep-mask and with its additive
    mask, in microseconds per call: back-to-back calls through the public API
    on one stream (CUDA events; the host's argument checks and launches set the
    pace), the host time per call, and the device time per call (the same calls
    captured in a CUDA graph and replayed)."""
    from attention_forward_tmem_b200 import api
    q, k, v, keep, add = (t.to(device) for t in W.page_example_masks())
    out = torch.empty(2, 8, 32, 96, device=device)
    res = {}
    for kind, mt, m in (("none", api.MaskType.NONE, None), ("bool_keep", api.MaskType.BOOL_KEEP, keep),
                        ("additive", api.MaskType.ADDITIVE, add)):
        fn = lambda: api.attn_fwd(q, k, v, mask=m, mask_type=mt, qk_scale=0.125, out=out)  # noqa: E731
        for _ in range(20):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        for _ in range(calls):
            fn()
        e1.record()
        t1 = time.perf_counter()
        torch.cuda.synchronize()
        per = 1e3 * e0.elapsed_time(e1) / calls
        host = 1e6 * (t1 - t0) / calls
        # device time alone: 20 calls in a graph, replayed
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(20):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(10):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        dev_us = 1e3 * e0.elapsed_time(e1) / 200
        del g
        res[kind] = {"us_per_call": per, "host_us_per_call": host, "device_us_per_call": dev_us}
    api.device_status()
    res["note"] = ("V^T kernel + attention kernel per call, fp32 inputs / TF32 products; "
                   f"{calls} back-to-back calls; device time from a CUDA graph of 20 calls")
    return res


def keep_mask_throughput(device, timer, peaks):
    """bf16 at the causal GQA shapes (B 4, 32/8 heads, L 4096, D 128) with a
    random boolean keep-mask [1, 1, L, L] (p_keep 0.8) read by the kernel.
    The metric counts kept pairs (the FLOP definition for masks); every tile
    is computed, so the rate over all L*L pairs is given beside it."""
    from attention_forward_tmem_b200 import api
    w = W.WORKLOADS["gqa_causal_prefill"]
    q, k, v = (t.to(device) for t in W.dense_inputs(w.batch, w.head_num, w.kv_head_num, w.seq, w.seq,
                                                     w.dqk, w.dv, w.dtype, W.SEED))
    g = torch.Generator(device="cpu")
    g.manual_seed(W.SEED)
    keep = (torch.rand(1, 1, w.seq, w.seq, generator=g) < 0.8).to(device)
    out = torch.empty_like(q)
    per_pair = w.batch * w.head_num * 2 * (w.dqk + w.dv)
    flops_all = per_pair * w.seq * w.seq
    flops_kept = per_pair * int(keep.sum().item())
    fn = lambda: api.attn_fwd(q, k, v, mask=keep, mask_type=api.MaskType.BOOL_KEEP,  # noqa: E731
                              qk_scale=w.qk_scale, out=out)
    ms, blocks, _, clocks = timer.run(fn)
    api.device_status()
    tf = flops_kept / (ms / 1e3) / 1e12
    tf_all = flops_all / (ms / 1e3) / 1e12
    return {"value": tf, "unit": "TFLOP/s (kept pairs)", "all_pairs_tflops": tf_all,
            "ms_per_step": ms, "timed_blocks": blocks,
            "frac_of_peak": tf_all / peaks["bf16_tflops_sustained"], "clocks": clocks,
            "config": "B 4, 32/8 heads, L 4096, D 128, bf16, keep-mask [1,1,4096,4096] p_keep 0.8 "
                      "(every tile computed; frac_of_peak over all pairs)"}


EXTRA_WORKLOADS = ["mla_varlen_prefill", "blockkv_rolling", "long_gqa_causal"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gqa_causal_prefill",
                    choices=["gqa_causal_prefill", "mla_varlen_prefill", "long_gqa_causal",
                             "blockkv_rolling"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the block of --steps timed steps until this much device time is timed")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-step-s", type=float, default=0.0,
                    help="reference arm: seconds of oracle work per step (0: from --ref-total-s)")
    ap.add_argument("--ref-total-s", type=float, default=150.0,
                    help="reference arm: target seconds for warm-up plus timed steps")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="dense workloads: a shorter sequence of the same shape (profiling cases)")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the headline workload only (no e2e, CPU baseline, other workloads or "
                         "comparison loop; for profilers)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        reference_arm(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return

    dist_on, rank, world = dist_setup(args)
    device = torch.device("cuda", torch.cuda.current_device())
    timer = BlockTimer(args.steps, args.warmup, args.min_timed_s, dist_on)
    peaks, peak_kind = measured_peaks()

    wl = make_workload(args.workload, device, args.seq_len)
    wl.to_device()
    headline_config = dict(wl.config)
    ms, blocks, total_ms, clocks, extra = measure(wl, timer, args)
    ms = parallel.max_over_ranks(ms, device)
    value = wl.flops * world / (ms / 1e3) / 1e12
    roofline = roofline_of(wl, ms, peaks, peak_kind)
    achieved = roofline["achieved"]

    e2e_val = h2d = d2h = None
    if not args.no_extras:
        e2e_steps = max(3, min(args.steps, 20))
        e2e_ms, h2d, d2h = time_e2e(wl, e2e_steps, 3)
        e2e_ms = parallel.max_over_ranks(e2e_ms, device)
        e2e_val = wl.flops * world * e2e_steps / (e2e_ms / 1e3) / 1e12
    headline_launches = args.steps * blocks * wl.launches_per_step
    del wl
    torch.cuda.empty_cache()

    # The other bf16 configurations (single GPU only): the same timing, one
    # entry each.
    workloads = None
    if not args.no_extras and world == 1:
        workloads = {}
        for name in EXTRA_WORKLOADS:
            if name == args.workload:
                continue
            w2 = make_workload(name, device)
            w2.to_device()
            ms2, blocks2, total2, clocks2, extra2 = measure(w2, timer, args)
            rl = roofline_of(w2, ms2, peaks, peak_kind)
            workloads[name] = dict({"value": rl["achieved"], "unit": "TFLOP/s", "ms_per_step": ms2,
                                    "steps": args.steps, "timed_blocks": blocks2,
                                    "timed_s": total2 / 1e3, "config": config_of(name),
                                    "roofline": rl, "clocks": clocks2,
                                    "gpu_launches": args.steps * blocks2 * w2.launches_per_step},
                                   **extra2)
            del w2
            torch.cuda.empty_cache()
        workloads["keep_mask_gqa_shapes"] = keep_mask_throughput(device, timer, peaks)
        torch.cuda.empty_cache()
        workloads["page_example_latency_us"] = page_example_latency(device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.no_extras:
        v, threads, note, _ = oracle_sample(args.workload)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": note}

    if dist_on:
        torch.distributed.barrier()
    if rank == 0:
        cfg = headline_config
        cfg["parallelism"] = f"dp{world}" if world > 1 else "single GPU"
        cfg["l2"] = "inputs larger than L2 (no flush needed)"
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "timed_blocks": blocks, "timed_s": total_ms / 1e3,
                "timing": (f"blocks of exactly {args.steps} steps, each bracketed by barrier + "
                           f"synchronize and timed by CUDA events, repeated until >= "
                           f"{args.min_timed_s} s was timed; ms_per_step = median block / steps"),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (seeded N(0,1), see workloads.py)",
                "config": cfg,
                "pct_of_peak": {"bf16_sustained": 100 * achieved / peaks["bf16_tflops_sustained"],
                                "bf16_burst": 100 * achieved / peaks["bf16_tflops"],
                                "datasheet_bf16_2250": 100 * achieved / DATASHEET_BF16_TFLOPS},
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "clocks": clocks,
                "gpu_launches": headline_launches}
        line.update(extra)
        if workloads is not None:
            line["workloads"] = workloads
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
