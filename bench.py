#!/usr/bin/env python
"""Benchmark of the HGA attention layer on B200.

Workloads (synthetic Qwen3-8B-shaped layers: 32 query heads, 8 KV heads,
head_dim 128, bf16, chunk 64, query block 64; seeded inputs drawn on the GPU
with the recipe of inputs/gen.py):

* ``qwen3_16k_fwd`` (default headline): 14,336 detached history tokens + a
  2,048-token active segment, top-16 chunks.  One step = route the 32 query
  blocks, exact-token attention forward over the routed chunks + the causal
  segment, and the detach-time summary append of the segment's 32 chunks.
* ``qwen3_16k_train``: the same layer trained segment-wise: one step = 8
  consecutive 2,048-token segments, each route + forward + backward (dQ, and
  dK/dV of the segment) + summary append.
* ``qwen3_128k_eval``: one step = a 131,072-token evaluation as 32 segments of
  4,096 tokens, top-32 chunks, each route + forward + summary append.
* ``qwen3_128k_tiered``: the 128K evaluation with detached history K/V in
  pinned host memory: each segment's route and the fetch of its routed chunks
  into a device staging cache run on a copy stream, under the attention of
  the segment before it (``hga_attn_fwd_tiered`` chained from segment to
  segment, one fetch wave of 64 query blocks per segment by default); the
  cache holds one segment's routing budget of chunk tiles and keeps them from
  segment to segment (it is emptied when the 131,072-token evaluation
  starts), so a routed chunk crosses the host link only when the cache does
  not hold it; the segment's K/V are offloaded to the host on a third stream
  (ordered before the next segment's fetches) and its summaries appended on
  the copy stream.
* ``qwen3_128k_decode``: generation at 128K context: 16 sequences each add one
  token after 131,008 detached history tokens; a step routes the 16 tokens
  (one-token query blocks) and runs the split-K decode attention over their 32
  routed chunks and 64-token local windows (query tok/s = tokens generated).
* ``qwen3_32k_decode``: the same decode step after 32,704 history tokens (the
  decode grid of the 128K case on 2.1 GB of K/V; used for counter captures).
* ``qwen3_16k_fwd_sink``: ``qwen3_16k_fwd`` with a one-chunk attention-sink
  window (history chunk 0 always routed, the other 15 slots by score).

The default run prints one JSON line for the headline workload and measures
``qwen3_16k_train``, ``qwen3_128k_eval``, ``qwen3_128k_tiered`` and
``qwen3_128k_decode`` too, each under ``workloads`` in the same line with its own
roofline, kernels, e2e and CPU baseline (``--also none`` skips them).

Metric: query tokens/s (active query tokens processed per second, all heads),
device-timed with CUDA events around each step, L2 flushed (256 MiB write)
before every step.  Device-resident workloads capture one step as a CUDA graph
and replay it; the route and forward of a segment are one hga_route_attn_fwd
call.  Per-kernel times come from a second graph of the same step with events
between the library calls (route and forward then issued apart), replayed as
many times after the timed region.  The tiered workload runs eagerly.
Each segment's summary append, which reads only the segment's keys, runs on a
side stream next to the segment's route (``--serial-append``: after attention).
Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HGA attn query tok/s at 16K & 128K ctx; % of HBM / tensor-pipe roofline"
UNIT = "query tok/s"
CSRC = "hierarchical_sparse_long_b200/csrc/"
# the translation unit of each kernel (and the PTX wrappers it inlines): a stored
# ncu traffic figure stays valid while these sources are unchanged
KERNEL_SOURCES = {
    "attn_fwd": [CSRC + "attn_fwd_tc.cu", CSRC + "tc_ptx.cuh", CSRC + "tc_issue.cuh"],
    "attn_bwd": [CSRC + "attn_bwd_tc.cu", CSRC + "tc_ptx.cuh", CSRC + "tc_issue.cuh"],
    "route": [CSRC + "route.cu", CSRC + "tc_ptx.cuh"],
    "summaries": [CSRC + "summaries.cu"],
    "fetch": [CSRC + "tiered.cu"],
    "attn_decode": [CSRC + "decode.cu", CSRC + "tc_ptx.cuh"],
}
WORKLOADS = ("qwen3_16k_fwd", "qwen3_16k_train", "qwen3_128k_eval", "qwen3_128k_tiered", "qwen3_16k_fwd_sink",
             "qwen3_128k_decode", "qwen3_32k_decode")
ALSO_DEFAULT = ("qwen3_16k_train", "qwen3_128k_eval", "qwen3_128k_tiered", "qwen3_128k_decode")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--workload", default="qwen3_16k_fwd", choices=WORKLOADS)
    ap.add_argument("--also", default="auto",
                    help="comma-separated workloads measured after the headline one and reported under "
                         "`workloads` ('none' for none; 'auto': the 16K training, 128K evaluation and 128K "
                         "tiered workloads when the headline is the default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--serial-append", action="store_true",
                    help="run each segment's summary append after its attention on the main stream "
                         "(default: on a side stream, overlapped with the route)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--tier-wave", type=int, default=64, help="query blocks per fetch wave of the tiered workload")
    ap.add_argument("--tier-lag", type=int, default=2,
                    help="a tiered fetch wave waits for the attention this many waves back (2..4)")
    ap.add_argument("--tier-host-only", action="store_true",
                    help="tiered fetches read every chunk from the host history (default: the previous "
                         "segment's chunks from its K/V still in device memory)")
    ap.add_argument("--only-last-segment", action="store_true",
                    help="a step processes only the workload's last segment (its history summarised up "
                         "front): for counter captures of the longest launches with few launches before them")
    ap.add_argument("--cpu-procs", type=int, default=0,
                    help="oracle processes for the 128K samples (0: up to 8, bounded by the host's cores)")
    return ap.parse_args()


def dist_setup():
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def code_text(src):
    """C/C++/CUDA source with its comments removed and blank or trailing space dropped:
    what the compiler sees, so an edit of comments alone keeps a kernel's stored counters.
    String and character literals are kept whole (an inline-asm string may hold '//')."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def file_hash(paths):
    """Hash of the code (comments and blank lines dropped) of the given source files."""
    h = hashlib.sha256()
    for p in paths:
        fp = os.path.join(ROOT, p)
        if os.path.exists(fp):
            h.update(code_text(open(fp, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    fp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(fp):
        return json.load(open(fp)), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(kernel, workload):
    """Per-launch DRAM bytes from the committed ncu summary, while the kernel source is unchanged."""
    fp = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(fp):
        return None
    d = json.load(open(fp)).get(f"{kernel}:{workload}")
    if not d or d.get("source_hash") != file_hash(KERNEL_SOURCES.get(kernel, [])):
        return None
    return d.get("bytes_per_launch")


def cpu_info():
    """Host CPU model, logical CPUs and the CPUs this process may run on."""
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    return {"cpu_model": model, "nproc": os.cpu_count() or 1, "usable_cpus": usable}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"hga_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        rows = [ln.split(",") for ln in open(self.path).read().strip().splitlines() if ln.count(",") >= 8]
        os.unlink(self.path)
        num = lambda s: s.strip().replace(".", "", 1).isdigit()
        sm = [float(r[1]) for r in rows if num(r[1])]
        mx = [float(r[2]) for r in rows if num(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ algorithmic work per launch
def attn_fwd_flops(w, T):
    """4*D*(k_eff*c + i + 1) flop per query row and head."""
    keff = min(w.topk, T // w.chunk)
    S = w.seg_len
    return 4 * w.head_dim * (keff * w.chunk * S + S * (S + 1) / 2) * w.batch * w.n_q_heads


def attn_bwd_flops(w, T):
    """dQ: 6*D per attended key per row (S, dP, dQ); dK/dV: 8*D per causal segment pair (S^T, dP^T, dV, dK)."""
    keff = min(w.topk, T // w.chunk)
    S = w.seg_len
    pairs_hist = keff * w.chunk * S
    pairs_seg = S * (S + 1) / 2
    return (6 * (pairs_hist + pairs_seg) + 8 * pairs_seg) * w.head_dim * w.batch * w.n_q_heads


def route_bytes(w, T):
    """Algorithmic bytes of one route: the queries read once, every routable
    summary read once, the route table written."""
    nqb = w.seg_len // w.q_block
    return (w.batch * w.n_q_heads * w.seg_len * w.head_dim * 2 +
            w.batch * w.n_kv_heads * (T // w.chunk) * w.head_dim * 4 +
            w.batch * w.n_kv_heads * nqb * w.topk * 4)


def summaries_bytes(w):
    return w.batch * w.n_kv_heads * w.seg_len * w.head_dim * 2 + \
        w.batch * w.n_kv_heads * (w.seg_len // w.chunk) * w.head_dim * 4


TILE_PAIR_BYTES = lambda w: 2 * w.chunk * w.head_dim * 2  # K and V of one chunk, bf16


# ------------------------------------------------------------------ workload state
class Layer:
    """Device state of one HGA layer: K/V of the whole sequence in one buffer per
    head (history and active segment are views), resident chunk summaries, and
    the queries (and upstream gradients) of every processed segment."""

    wave = 64  # query blocks per tiered fetch wave
    lag = 2  # a tiered fetch waits for the attention this many waves back
    prev_source = True  # tiered fetches copy the previous segment's chunks from its device K/V

    def __init__(self, w):
        import torch
        from inputs import gen
        import hierarchical_sparse_long_b200 as hga
        self.w, self.hga, self.torch = w, hga, torch
        L = w.seq_len
        self.L = L
        dev = torch.device("cuda")
        t0 = time.time()
        self.k = gen.keys_torch(w, 0, L, dev).contiguous()
        self.v = gen.values_torch(w, 0, L, dev).contiguous()
        self.q = {T: gen.queries_torch(w, T, T + w.seg_len, dev).contiguous() for T in w.seg_starts}
        self.do = {T: gen.grad_out_torch(w, T, T + w.seg_len, dev).contiguous() for T in w.seg_starts} \
            if w.backward else {}
        torch.cuda.synchronize()
        self.gen_seconds = time.time() - t0
        self.nct = L // w.chunk
        self.summ = torch.zeros(w.batch, w.n_kv_heads, self.nct, w.head_dim, device=dev)
        nqb = w.seg_len // w.q_block
        self.idx = torch.empty(w.batch, w.n_kv_heads, nqb, w.topk, device=dev, dtype=torch.int32)
        self.out = torch.empty(w.batch, w.n_q_heads, w.seg_len, w.head_dim, device=dev, dtype=torch.bfloat16)
        self.lse = torch.empty(w.batch, w.n_q_heads, w.seg_len, device=dev)
        if w.backward:
            self.dq = torch.empty(self.out.shape, device=dev)
            self.dk = torch.empty(w.batch, w.n_kv_heads, w.seg_len, w.head_dim, device=dev)
            self.dv = torch.empty_like(self.dk)
            self.ws = torch.empty(hga.hga_attn_bwd_workspace_size(self.params(w.seg_starts[-1])) // 4 + 64,
                                  device=dev)
        self.side = torch.cuda.Stream()
        self.side_append = False
        # a multi-segment forward-only evaluation: each segment's route (and append) on a
        # route stream, under the attention of the segment before it (hga_segment_fwd)
        self.pipelined = not w.backward and not w.tiered and len(w.seg_starts) > 1
        if self.pipelined:
            self.route_stream = torch.cuda.Stream(priority=-1)
            self.idx_ring = [self.idx, torch.empty_like(self.idx)]
            self.sched = hga.TierSched(lag=2)
        if w.tiered:
            self._init_tiered()
        self.reset()

    def reset(self):
        """Summaries of the history that exists before the first processed segment."""
        w = self.w
        self.summ.zero_()
        first = w.seg_starts[0] // w.chunk
        if first:
            self.hga.hga_build_summaries(self.k, self.L, w.batch, w.n_kv_heads, w.head_dim, w.chunk, 0, first,
                                         self.summ, self.nct)

    def params(self, T, **kw):
        w = self.w
        p = self.hga.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                            topk=w.topk, seg_len=w.seg_len, n_hist_chunks=T // w.chunk, dtype=self.hga.HGA_BF16,
                            hist_head_stride=self.L, seg_head_stride=self.L, chunk=w.chunk, q_block=w.q_block,
                            sink_chunks=w.sink_chunks)
        for k, v in kw.items():
            setattr(p, k, v)
        return p

    def segment(self, T, ev=None, q=None, do=None, si=0, outs=None):
        """Route, attend [, backward], detach with history in device memory;
        returns the number of library kernels launched.  Uninstrumented (ev is
        None), the route and the forward are one hga_route_attn_fwd call, or,
        in a multi-segment forward-only evaluation, one hga_segment_fwd call
        whose route runs on a route stream under the previous segment's
        attention (its q, K and V are then resident or were copied in on the
        route stream).

        With side_append the detach-time summary append (it reads only the
        segment's keys and writes summaries of chunks this segment's route
        never reads) runs on a side stream next to the route, whose grid leaves
        SMs free, and is joined before the segment ends."""
        torch, hga, w = self.torch, self.hga, self.w
        p = self.params(T)
        q = self.q[T] if q is None else q
        ks, vs = self.k[:, :, T:], self.v[:, :, T:]
        # the segment's outputs: O, LSE [, dQ, dK, dV]
        o_out, o_lse, o_dq, o_dk, o_dv = outs if outs is not None else (
            self.out, self.lse, getattr(self, "dq", None), getattr(self, "dk", None), getattr(self, "dv", None))
        if ev is None and self.pipelined:
            hga.hga_segment_fwd(p, q, self.k, self.v, ks, vs, self.summ, self.nct, self.idx_ring[si % 2], o_out,
                                o_lse, self.sched, reset=si == 0, route_stream=self.route_stream)
            return 3  # route, forward, append
        rec = ev.record if ev is not None else (lambda name: None)
        main = torch.cuda.current_stream()
        if self.side_append:
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                if ev is not None:
                    ev.record("summaries")
                hga.hga_build_summaries(self.k, self.L, w.batch, w.n_kv_heads, w.head_dim, w.chunk, T // w.chunk,
                                        w.seg_len // w.chunk, self.summ, self.nct)
                if ev is not None:
                    ev.record(None)
        if ev is None:
            hga.hga_route_attn_fwd(p, q, self.summ, self.nct, self.idx, self.k, self.v, ks, vs, o_out, o_lse)
        else:
            rec("route")
            hga.hga_route(p, q, self.summ, self.nct, self.idx)
            rec("attn_fwd")
            hga.hga_attn_fwd(p, q, self.k, self.v, ks, vs, self.idx, o_out, o_lse)
        launches = 2
        if w.backward:
            rec("attn_bwd")
            hga.hga_attn_bwd(p, q, self.k, self.v, ks, vs, self.idx, o_out, o_lse,
                             self.do[T] if do is None else do, o_dq, o_dk, o_dv, self.ws)
            launches += 2
        if self.side_append:
            rec(None)
            main.wait_stream(self.side)
        else:
            rec("summaries")
            hga.hga_build_summaries(self.k, self.L, w.batch, w.n_kv_heads, w.head_dim, w.chunk, T // w.chunk,
                                    w.seg_len // w.chunk, self.summ, self.nct)
            rec(None)
        return launches + 1

    def _init_tiered(self):
        """Pinned host copy of the whole sequence's K/V (the detached history is
        read from there only) and the device staging cache: one segment's routing
        budget of chunk tiles (as many tiles as the segment's blocks can route to)."""
        torch, hga, w = self.torch, self.hga, self.w
        self.host_k = self.k.cpu().pin_memory()
        self.host_v = self.v.cpu().pin_memory()
        nqb = w.seg_len // w.q_block
        self.slots = w.batch * w.n_kv_heads * min(w.seg_starts[-1] // w.chunk, nqb * w.topk)
        self.stage_k = torch.empty(self.slots, w.chunk, w.head_dim, device="cuda", dtype=torch.bfloat16)
        self.stage_v = torch.empty_like(self.stage_k)
        p0 = self.params(w.seg_starts[-1])
        self.scratch = torch.empty(hga.hga_tier_scratch_size(p0, self.slots) // 4, device="cuda",
                                   dtype=torch.int32)
        self.n_waves = -(-nqb // self.wave)
        # the fetch of a wave rewrites its blocks' remapped routes once the attention
        # `lag` waves back is done: chained segments rotate enough buffers
        self.idx_r = [torch.empty_like(self.idx) for _ in range(-(-self.lag // self.n_waves))]
        # a route may run a segment ahead of the fetches that read the one before it
        self.idx_ring = [self.idx, torch.empty_like(self.idx)]
        self.n_fetched = torch.zeros(len(w.seg_starts), self.n_waves, device="cuda", dtype=torch.int32)
        # the side streams' kernels are small; at high priority they take SMs as the
        # attention's CTAs retire instead of waiting behind the whole attention grid
        self.copy_stream = torch.cuda.Stream(priority=-1)
        self.route_stream = torch.cuda.Stream(priority=-1)
        self.offload_stream = torch.cuda.Stream(priority=-1)
        self.sched = hga.TierSched(lag=self.lag)

    def segment_tiered(self, T, ev=None, q=None, si=0, outs=None):
        """The same segment with the history only in pinned host memory, one
        hga_segment_fwd_tiered call on four streams: the route and the summary
        append on a route stream, the fetch of the routed tiles on a copy stream
        (chained from segment to segment over the staging cache, the cache emptied
        at the first segment only), the segment's K/V offload to the host history
        on a third, the attention on the compute stream -- so a segment's route
        and fetches run under the attention of the segments before it.  The
        segment's q, K and V are resident, or were copied in on the route stream."""
        hga, w = self.hga, self.w
        p = self.params(T)
        q = self.q[T] if q is None else q
        ks, vs = self.k[:, :, T:], self.v[:, :, T:]
        # the previous segment's K/V are still in device memory: its chunks are
        # copied from there rather than back across the host link
        prev = si > 0 and self.prev_source and T >= w.seg_len
        pk = self.k[:, :, T - w.seg_len:] if prev else None
        pv = self.v[:, :, T - w.seg_len:] if prev else None
        if ev is not None:
            ev.record("attn_fwd")
        first = si == 0
        hga.hga_segment_fwd_tiered(p, q, ks, vs, self.summ, self.nct, self.idx_ring[si % 2], self.host_k,
                                   self.host_v, self.out if outs is None else outs[0],
                                   self.lse if outs is None else outs[1], self.stage_k, self.stage_v, self.slots,
                                   self.scratch, self.idx_r[si % len(self.idx_r)], self.wave, self.sched,
                                   reset=first, n_fetched=self.n_fetched[si], copy_stream=self.copy_stream,
                                   route_stream=self.route_stream, offload_stream=self.offload_stream,
                                   prev_k_seg=pk, prev_v_seg=pv)
        if ev is not None:
            ev.record(None)
        # route, reset (first segment), fetch waves (plan, copy, remap) + attention, append
        return 1 + int(first) + (1 if T == 0 else 4 * self.n_waves) + 1

    def end_tiered_step(self):
        """The step ends when the side streams' work (the last append and offload) has."""
        compute = self.torch.cuda.current_stream()
        compute.wait_stream(self.copy_stream)
        compute.wait_stream(self.route_stream)
        compute.wait_stream(self.offload_stream)

    def fetch_only_step(self):
        """Route + every fetch wave of every segment on the copy stream, no attention
        and no offload (the host-link side of the tiered step alone, the cache emptied
        at the first segment as in the step); returns device ms."""
        torch, hga, w = self.torch, self.hga, self.w
        compute = torch.cuda.current_stream()
        nqb = w.seg_len // w.q_block
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(compute)
        for si, T in enumerate(w.seg_starts):
            p = self.params(T)
            hga.hga_route(p, self.q[T], self.summ, self.nct, self.idx)
            if T == 0:
                continue
            self.copy_stream.wait_stream(compute)
            if T == w.seg_starts[0] or (si == 1 and w.seg_starts[0] == 0):  # the step's first fetch
                hga.hga_tier_reset(p, self.slots, self.scratch, stream=self.copy_stream)
            for wi, b0 in enumerate(range(0, nqb, self.wave)):
                hga.hga_fetch_tiered(p, self.host_k, self.host_v, self.idx, b0, min(b0 + self.wave, nqb),
                                     self.stage_k, self.stage_v, self.slots, self.scratch, self.idx_r[0],
                                     self.n_fetched[si, wi:wi + 1], copy_stream=self.copy_stream)
            compute.wait_stream(self.copy_stream)
        e.record(compute)
        e.synchronize()
        return s.elapsed_time(e)

    def distinct_tiles(self):
        """Distinct (b, g, chunk) tiles each segment routes to, summed over the
        segments (what a cache emptied at every segment would fetch), and over the
        whole step (what an unbounded cache would fetch).  Runs the routes again on
        the same summaries; not timed."""
        torch, hga, w = self.torch, self.hga, self.w
        total, seen = 0, []
        for T in w.seg_starts:
            if T == 0:
                continue
            hga.hga_route(self.params(T), self.q[T], self.summ, self.nct, self.idx)
            bg = torch.arange(w.batch * w.n_kv_heads, device="cuda").view(w.batch, w.n_kv_heads, 1, 1)
            keys = torch.unique((bg * self.nct + self.idx.long())[self.idx >= 0])
            total += int(keys.numel())
            seen.append(keys)
        return total, int(torch.unique(torch.cat(seen)).numel()) if seen else 0

    def step(self, ev=None):
        # the summaries of chunks >= T are never read by the route of a segment
        # starting at T, so each step simply re-appends every segment's chunks
        n = 0
        for si, T in enumerate(self.w.seg_starts):
            n += self.segment_tiered(T, ev, si=si) if self.w.tiered else self.segment(T, ev, si=si)
        if self.w.tiered:  # the last append and offload belong to the step
            self.end_tiered_step()
        elif self.pipelined and ev is None:  # the last append belongs to the step
            self.torch.cuda.current_stream().wait_stream(self.route_stream)
        return n


class PhaseEvents:
    """CUDA events on the launching (current) stream between the phases of a
    step.  With external=True the events become event-record nodes when the
    step is captured into a CUDA graph, and every replay re-records them."""

    def __init__(self, external=False):
        import torch
        self.torch = torch
        self.external = external
        self.marks = {}  # per stream: [(phase name or None, event)]

    def record(self, name):
        stream = self.torch.cuda.current_stream()
        e = self.torch.cuda.Event(enable_timing=True, external=self.external)
        e.record(stream)
        self.marks.setdefault(stream.cuda_stream, []).append((name, e))

    def totals(self):
        out = {}
        for marks in self.marks.values():
            for (name, a), (_, b) in zip(marks, marks[1:]):
                if name is not None:
                    out[name] = out.get(name, 0.0) + a.elapsed_time(b)
        return out


def flush_l2(buf):
    buf.add_(1)


def max_over_ranks(ms, world, device):
    """The slowest rank's device time (every rank calls this, in the same order)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step, steps, world, total_ms):
    """Whole-job query tokens/s: every rank processes its own layer instance
    (weak scaling), timed by the slowest rank."""
    return tokens_per_step * steps * world / (total_ms / 1000.0)


# ------------------------------------------------------------------ CPU oracle sample
def tokens_per_step(w):
    """Query tokens a step processes: one per sequence when decoding."""
    return w.batch if w.decode else w.seg_len * w.batch * len(w.seg_starts)


def workload_config(w, world):
    """The workload keys of the JSON line's `config`, the same for both arms."""
    cfg = {"workload": w.name, "batch": w.batch, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
           "head_dim": w.head_dim, "context": w.seq_len}
    if w.decode:
        cfg.update({"history_tokens": w.seg_starts[0], "local_window": w.seg_len, "topk": w.topk,
                    "sink_chunks": w.sink_chunks, "chunk": w.chunk, "decode": True,
                    "tokens_per_step": tokens_per_step(w)})
    else:
        cfg.update({"seg_len": w.seg_len, "topk": w.topk, "sink_chunks": w.sink_chunks, "chunk": w.chunk,
                    "q_block": w.q_block, "segments_per_step": len(w.seg_starts), "backward": w.backward,
                    "tiered": w.tiered})
    cfg["parallelism"] = f"one independent layer per GPU x{world}"
    return cfg


def decode_oracle_sample(w, target_seconds):
    """The oracle on the decode token of sequence 0 (its inputs drawn alone with the same
    generator): its route (the oracle routes every token of the local window as a one-token
    block; that time is divided by the window length) and its attention."""
    import dataclasses

    import numpy as np

    import oracle
    from inputs import gen
    w1 = dataclasses.replace(w, batch=1)  # element n of sequence 0 is the same in a batch-1 draw
    T, L, D = w.seg_starts[0], w.seg_len, w.head_dim
    q = gen.queries_torch(w1, T, T + L, "cpu").float().numpy()
    k_all = gen.keys_torch(w1, 0, T + L, "cpu").float().numpy()
    v_all = gen.values_torch(w1, 0, T + L, "cpu").float().numpy()
    sh = oracle.shape(1, w.n_q_heads, w.n_kv_heads, D, w.chunk, 1, w.topk, L, T // w.chunk, w.sink_chunks)
    summ = oracle.summaries(k_all[:, :, :T], w.chunk)
    reps, t_route, t_attn = 0, 0.0, 0.0
    while reps == 0 or (t_route + t_attn < target_seconds and reps < 50):
        t0 = time.perf_counter()
        idx, _, _ = oracle.route(sh, q, summ)
        t_route += (time.perf_counter() - t0) / L
        rows = np.array([h * L + L - 1 for h in range(w.n_q_heads)], dtype=np.int64)
        t0 = time.perf_counter()
        oracle.attn_fwd(sh, q, k_all[:, :, :T], v_all[:, :, :T], k_all[:, :, T:], v_all[:, :, T:], idx, rows=rows)
        t_attn += time.perf_counter() - t0
        reps += 1
    per_token = (t_route + t_attn) / reps
    desc = (f"oracle fp64 single-thread, decode token of sequence 0 ({T} history tokens, {L}-token window): "
            f"route (window routes / {L}) + attention, {reps} repetitions; history summaries not counted")
    return 1.0 / per_token, desc, 1


def _oracle_block_task(task):
    """One sampled query block through the oracle (a worker of the CPU baseline):
    forward of the block's rows for every head and, when dO is given, the backward's
    dQ rows of the same block.  The routed chunks of the block arrive gathered in
    route order, so the oracle runs the same arithmetic as on the whole history.
    Returns (forward seconds, backward seconds)."""
    import numpy as np

    import oracle
    shp, m, q_blk, kh, vh, ks, vs, idx, do_blk = task
    B, Hq, _, D = q_blk.shape
    S = ks.shape[2]
    q = np.zeros((B, Hq, S, D), dtype=np.float32)
    q[:, :, m * 64:(m + 1) * 64] = q_blk
    rows = np.array([(b * Hq + h) * S + m * 64 + i for b in range(B) for h in range(Hq) for i in range(64)],
                    dtype=np.int64)
    sh = oracle.shape(*shp)
    t0 = time.perf_counter()
    oracle.attn_fwd(sh, q, kh, vh, ks, vs, idx, rows=rows)
    t_f = time.perf_counter() - t0
    t_b = 0.0
    if do_blk is not None:
        do = np.zeros_like(q)
        do[:, :, m * 64:(m + 1) * 64] = do_blk
        q_need = np.zeros((B, Hq, S), dtype=np.uint8)
        q_need[:, :, m * 64:(m + 1) * 64] = 1
        key_need = np.zeros((B, ks.shape[1], S), dtype=np.uint8)
        t0 = time.perf_counter()
        oracle.attn_bwd(sh, q, kh, vh, ks, vs, idx, do, q_need=q_need, key_need=key_need)
        t_b = time.perf_counter() - t0
    return t_f, t_b


def oracle_sample(w, target_seconds, procs=1):
    """Times the CPU oracle on a bounded sample of the workload and projects it to one
    step; returns (tok/s, cpu_baseline dict)."""
    info = cpu_info()
    if w.decode:
        tok_s, desc, cores = decode_oracle_sample(w, target_seconds)
        return tok_s, {"cores": cores, "sample": desc, **info}
    import numpy as np

    import oracle
    from inputs import gen
    T = w.seg_starts[-1]
    S, D, B = w.seg_len, w.head_dim, w.batch
    nqb = S // w.q_block
    q = gen.queries_torch(w, T, T + S, "cpu").float().numpy()
    k_all = gen.keys_torch(w, 0, T + S, "cpu").float().numpy()
    v_all = gen.values_torch(w, 0, T + S, "cpu").float().numpy()
    do = gen.grad_out_torch(w, T, T + S, "cpu").float().numpy() if w.backward else None
    sh = oracle.shape(B, w.n_q_heads, w.n_kv_heads, D, w.chunk, w.q_block, w.topk, S, T // w.chunk, w.sink_chunks)
    t0 = time.perf_counter()
    oracle.summaries(k_all[:, :, T:], w.chunk)  # detach-time summaries of the segment
    t_summ = time.perf_counter() - t0
    summ = oracle.summaries(k_all[:, :, :T], w.chunk) if T else np.zeros((B, w.n_kv_heads, 0, D))
    t0 = time.perf_counter()
    idx, _, _ = oracle.route(sh, q, summ)
    t_route = time.perf_counter() - t0
    keff = min(w.topk, T // w.chunk)
    ks, vs = np.ascontiguousarray(k_all[:, :, T:]), np.ascontiguousarray(v_all[:, :, T:])

    def task(m):
        # the block's routed chunks gathered in route order: chunk slot a of head g
        kh = np.zeros((B, w.n_kv_heads, max(keff, 1) * w.chunk, D), dtype=np.float32)
        vh = np.zeros_like(kh)
        ic = np.full(idx.shape, -1, dtype=np.int32)
        for b in range(B):
            for g in range(w.n_kv_heads):
                for a, j in enumerate(idx[b, g, m]):
                    if j >= 0:
                        kh[b, g, a * w.chunk:(a + 1) * w.chunk] = k_all[b, g, j * w.chunk:(j + 1) * w.chunk]
                        vh[b, g, a * w.chunk:(a + 1) * w.chunk] = v_all[b, g, j * w.chunk:(j + 1) * w.chunk]
                        ic[b, g, m, a] = a
        shp = (B, w.n_q_heads, w.n_kv_heads, D, w.chunk, w.q_block, w.topk, S, max(keff, 1), 0)
        d_blk = do[:, :, m * 64:(m + 1) * 64] if do is not None else None
        return shp, m, q[:, :, m * 64:(m + 1) * 64].copy(), kh, vh, ks, vs, ic, d_blk

    # blocks spread over the segment, latest (most keys) first
    order = list(range(nqb - 1, -1, -max(1, nqb // 8)))
    times, blocks = [], []
    t_wall0 = time.perf_counter()
    if procs <= 1:
        for m in order:
            times.append(_oracle_block_task(task(m)))
            blocks.append(m)
            if sum(a + b for a, b in times) + t_route > target_seconds:
                break
    else:
        import concurrent.futures
        import multiprocessing
        n_tasks = min(len(order), procs * max(1, int(target_seconds // 8)))
        blocks = sorted({order[int(i * len(order) / n_tasks)] for i in range(n_tasks)}, reverse=True)
        ctx = multiprocessing.get_context("spawn")  # never fork a process that has used the GPU
        with concurrent.futures.ProcessPoolExecutor(max_workers=procs, mp_context=ctx) as ex:
            t_wall0 = time.perf_counter()
            times = list(ex.map(_oracle_block_task, [task(m) for m in blocks]))
    t_wall = time.perf_counter() - t_wall0
    t_fwd = sum(a for a, _ in times)
    t_bwd = sum(b for _, b in times)
    # attention work of a block ~ attended keys per row: k_eff*c + m*64 + 32.5
    cost = lambda kf, m: kf * w.chunk + m * w.q_block + (w.q_block + 1) / 2
    per_cost_f = t_fwd / sum(cost(keff, m) for m in blocks)
    per_cost_b = t_bwd / sum(cost(keff, m) for m in blocks)
    core_s = 0.0
    route_s = 0.0
    for Ts in w.seg_starts:  # project to every segment of the step
        kf = min(w.topk, Ts // w.chunk)
        core_s += sum(cost(kf, m) for m in range(nqb)) * (per_cost_f + per_cost_b)
        route_s += t_route * (Ts / T if T else 0.0) + t_summ
    cores = max(1, procs)
    step_s = core_s / cores + route_s
    tok_s = tokens_per_step(w) / step_s
    what = "forward" + (" + backward dQ rows (dK/dV accumulation not timed)" if w.backward else "")
    desc = (f"oracle fp64, {cores} process(es) of one thread: summaries + route of the last {S}-token segment "
            f"(T={T}) and the {what} of query blocks {sorted(blocks)} (all {w.n_q_heads} heads), projected by "
            f"attended-key count to all {len(w.seg_starts)} segment(s) of a step; blocks sharded over the "
            f"processes, route and summaries on one; sample {sum(a + b for a, b in times) + t_route:.1f} "
            f"core-s in {t_wall + t_route:.1f} s wall")
    return tok_s, {"cores": cores, "sample": desc, "core_seconds_per_step": round(core_s + route_s, 2),
                   "wall_seconds_per_step": round(step_s, 3), **info}


# ------------------------------------------------------------------ arms
def run_reference(args, rank):
    from inputs import gen
    if rank != 0:
        return
    w = gen.WORKLOADS[args.workload]
    import oracle
    oracle.build()
    budget = max(2.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    per_step, cb, walls = [], {}, []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        tok_s, cb = oracle_sample(w, budget)
        walls.append((time.perf_counter() - t0) * 1000)
        if s >= args.warmup:
            per_step.append(tok_s)
    v = statistics.median(per_step)
    ms = tokens_per_step(w) / v * 1000
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "step_is_sample": "each step times a bounded sample of the workload on the host cores; value and "
                              "ms_per_step are that sample projected to a whole step",
            "sample_wall_ms_per_step": round(statistics.median(walls[args.warmup:]), 1),
            "cpu_baseline": {"value": v, "unit": UNIT, "kind": "oracle", **cb},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def host_link_gbs(nbytes=256 << 20):
    """Pinned host <-> device copy bandwidth measured here (the tiered path's roofline):
    host -> device alone, device -> host alone, and both directions at once (two
    streams; the sum of the bytes over the time of the pair), each the best of five."""
    import torch
    h_in = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    h_out = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    d_out = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def best(h2d, d2h):
        top = 0.0
        for _ in range(6):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(main)
            s_in.wait_stream(main)
            s_out.wait_stream(main)
            if h2d:
                with torch.cuda.stream(s_in):
                    d_in.copy_(h_in, non_blocking=True)
            if d2h:
                with torch.cuda.stream(s_out):
                    h_out.copy_(d_out, non_blocking=True)
            main.wait_stream(s_in)
            main.wait_stream(s_out)
            e.record(main)
            e.synchronize()
            top = max(top, (int(h2d) + int(d2h)) * nbytes / (s.elapsed_time(e) / 1000) / 1e9)
        return top

    return {"h2d": best(True, False), "d2h": best(False, True), "both": best(True, True)}


def measure_layer(w, args, world, local):
    """Times one device-resident or tiered workload; returns its JSON fields."""
    import torch
    import hierarchical_sparse_long_b200 as hga
    Layer.wave = args.tier_wave
    Layer.lag = args.tier_lag
    Layer.prev_source = not args.tier_host_only
    if args.only_last_segment:
        import dataclasses
        w = dataclasses.replace(w, seg_starts=w.seg_starts[-1:])
    layer = Layer(w)
    layer.side_append = not args.serial_append and not w.tiered
    flush = torch.empty(256 * 1024 * 1024 // 4, device="cuda", dtype=torch.float32)
    for _ in range(args.warmup):
        flush_l2(flush)
        layer.step()
    torch.cuda.synchronize()
    bits = hga.hga_get_device_status()
    if bits != 0:
        raise RuntimeError(f"{w.name}: device status bits {bits:#x} during warm-up")
    # Device-resident workloads replay one step captured as a CUDA graph (one
    # host launch per step; the route and the forward in one call, the forward
    # overlapping the route's tail); the tiered workload drives its copy stream
    # from the host and stays eager.  A second graph of the same step with CUDA
    # events between the library calls (issued apart) gives the per-kernel
    # times, replayed after the timed region: event nodes inside the timed
    # graph would add their own gaps to the step.
    graph, pgraph, gev = None, None, None
    if not w.tiered:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            graph_launches = layer.step()
        gev = PhaseEvents(external=True)
        pgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pgraph):
            layer.step(ev=gev)
        for gr in (graph, pgraph):
            flush_l2(flush)
            gr.replay()
        torch.cuda.synchronize()
    sampler = ClockSampler(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    phases = []
    launches = 0
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for s in range(args.steps):
        flush_l2(flush)
        starts[s].record()
        if graph is not None:
            graph.replay()
            launches += graph_launches
        else:
            launches += layer.step()
        ends[s].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(starts, ends)), world, "cuda")
    value = job_throughput(tokens_per_step(w), args.steps, world, total_ms)
    # per-kernel device times: the instrumented step, as many times as the timed one
    for s in range(args.steps):
        flush_l2(flush)
        if pgraph is not None:
            pgraph.replay()
            torch.cuda.synchronize()
            phases.append(gev.totals())
        else:
            ev = PhaseEvents()
            layer.step(ev=ev)
            phases.append(ev)
    torch.cuda.synchronize()
    status = hga.hga_get_device_status()

    # per-kernel device time over the timed steps (events on the launching stream)
    ph = {}
    for ev in phases:
        for k, v in (ev if isinstance(ev, dict) else ev.totals()).items():
            ph[k] = ph.get(k, 0.0) + v
    n_seg = len(w.seg_starts) * args.steps
    peaks, peak_src = measured_peaks()
    fwd_fl = sum(attn_fwd_flops(w, T) for T in w.seg_starts) * args.steps
    kernels = {
        "attn_fwd": {"bound": "tensor", "ms_per_launch": ph["attn_fwd"] / n_seg,
                     "achieved": fwd_fl / (ph["attn_fwd"] / 1e3) / 1e12, "unit": "TFLOP/s"},
    }
    if "route" in ph:
        kernels["route"] = {"bound": "hbm", "ms_per_launch": ph["route"] / n_seg,
                            "achieved": sum(route_bytes(w, T) for T in w.seg_starts) * args.steps /
                            (ph["route"] / 1e3) / 1e9, "unit": "GB/s"}
    if "summaries" in ph:
        kernels["summaries"] = {"bound": "hbm", "ms_per_launch": ph["summaries"] / n_seg,
                                "achieved": summaries_bytes(w) * n_seg / (ph["summaries"] / 1e3) / 1e9,
                                "unit": "GB/s"}
    if layer.side_append:
        kernels["summaries"]["note"] = "on a side stream, timed while it overlaps the route"
    if w.tiered:
        kernels["attn_fwd"]["note"] = "the compute stream's share of hga_segment_fwd_tiered: the attention " \
                                      "waves and the waits for the fetches they cannot hide (the route, " \
                                      "fetches, append and offload run on two side streams)"
    if w.backward:
        bwd_fl = sum(attn_bwd_flops(w, T) for T in w.seg_starts) * args.steps
        kernels["attn_bwd"] = {"bound": "tensor", "ms_per_launch": ph["attn_bwd"] / n_seg,
                               "achieved": bwd_fl / (ph["attn_bwd"] / 1e3) / 1e12, "unit": "TFLOP/s"}
    for k, v in kernels.items():
        pk = peaks["bf16_tflops"] if v["unit"] == "TFLOP/s" else peaks["hbm_gbs"]
        v["frac"] = round(v["achieved"] / pk, 4)
        v["achieved"] = round(v["achieved"], 2)
        v["ms_per_launch"] = round(v["ms_per_launch"], 4)
    dom = max((k for k in kernels if kernels[k]["bound"] == "tensor"), key=lambda k: ph[k])
    kd = kernels[dom]
    roof = {"bound": "tensor", "kernel": "hga_" + dom, "achieved": kd["achieved"], "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": kd["frac"], "traffic": kernel_traffic(dom, w.name),
            "peak_source": f"{peak_src}: MEASURED_PEAKS.json bf16_tflops (burst)",
            "units_per_launch": "4*D*(k_eff*64+i+1) flop per query row and head" if dom == "attn_fwd" else
            "dQ 6*D per attended key, dK/dV 8*D per causal segment pair, per row and head"}
    res = {"value": value, "unit": UNIT, "ms_per_step": total_ms / args.steps,
           "config": {**workload_config(w, world),
                      "l2": "flushed before every timed step (256 MiB write)",
                      "launch": "one CUDA graph replay per step" if graph is not None else "eager",
                      "route_and_forward": ("hga_segment_fwd_tiered (route on a route stream, fetches on a "
                                            "copy stream, chained across segments)" if w.tiered else
                                            "hga_segment_fwd (each segment's route on a route stream under "
                                            "the previous segment's attention)" if layer.pipelined else
                                            "hga_route_attn_fwd (one call, the forward a programmatic "
                                            "dependent of the route)"),
                      "kernel_times": "from as many replays of the same step with CUDA events between its "
                                      "library calls (route and forward then issued apart), after the "
                                      "timed region",
                      "append": ("route stream, overlapped with the attention" if w.tiered or layer.pipelined
                                 else "side stream, overlapped with the route" if layer.side_append
                                 else "in order")},
           "roofline": roof, "kernels": kernels, "clocks": clocks, "gpu_launches": launches,
           "device_status": status}
    if w.tiered:
        res["tiered"] = tiered_report(layer, total_ms / args.steps, ph["attn_fwd"] / args.steps, flush)
        # the step's dominant cost is the host link: its own roofline line
        t = res["tiered"]
        # the fetches (host -> device) and the detach copies (device -> host) share the
        # link: both directions' bytes over the step against both directions at once
        pk = t["host_link_gbs_measured"]["both"]
        res["roofline_host_link"] = {"bound": "host link", "achieved": t["link_both_gbs_achieved"],
                                     "peak": pk, "unit": "GB/s",
                                     "frac": round(t["link_both_gbs_achieved"] / pk, 4),
                                     "traffic": t["bytes_fetched_per_step"] + t["bytes_offloaded_per_step"],
                                     "peak_source": "pinned cudaMemcpyAsync host -> device and device -> host "
                                                    "at once on two streams, measured in this run"}
    single = len(w.seg_starts) == 1 and not w.backward and not w.tiered
    res["e2e"] = e2e_stream_measure(layer, max(10, args.steps)) if single else \
        e2e_measure(layer, max(2, min(args.steps, 5)))
    del layer, graph
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def tiered_report(layer, step_ms, attn_phase_ms, flush):
    """Host-link accounting of the tiered step: tiles fetched from the host per step
    (the previous segment's chunks come from device memory unless --tier-host-only)
    against the distinct tiles the segments route to, the fetch-only step (every
    chunk from the host) and the resident
    attention (no host link), and the share of the attention hidden under the
    fetches: (fetch-only + resident attention - tiered attention phase) /
    resident attention, the tiered phase being the fetch waves and attention of
    every segment on the compute stream's timeline."""
    import torch
    w = layer.w
    fetched = int(layer.n_fetched.sum().item())
    per_segment, whole = layer.distinct_tiles()
    flush_l2(flush)
    t_fetch = layer.fetch_only_step()
    # the attention alone with the history resident in device memory (no host link)
    ev = PhaseEvents()
    flush_l2(flush)
    for T in w.seg_starts:
        layer.segment(T, ev=ev)
    torch.cuda.synchronize()
    t_res = ev.totals()["attn_fwd"]
    link = host_link_gbs()
    tb = TILE_PAIR_BYTES(w)
    # the detach copies every segment's K/V to the host history: device -> host bytes
    off_b = len(w.seg_starts) * w.batch * w.n_kv_heads * w.seg_len * w.head_dim * 2 * 2
    hidden = (t_fetch + t_res - attn_phase_ms) / t_res if t_res > 0 else None
    return {"staging_slots": layer.slots, "staging_mib": round(layer.slots * tb / 2**20, 1),
            "cache_policy": "one segment's routing budget of chunk tiles, kept from segment to segment and "
                            f"emptied when the evaluation starts; waves of {layer.wave} query blocks, a fetch "
                            f"after the attention {layer.lag} waves back",
            "fetch_source": "host history; the previous segment's chunks from its K/V still in device memory"
                            if layer.prev_source else "host history for every chunk",
            "tiles_fetched_per_step": fetched, "tiles_distinct_per_segment_summed": per_segment,
            "tiles_distinct_per_step": whole,
            "bytes_fetched_per_step": fetched * tb, "bytes_distinct_per_segment_summed": per_segment * tb,
            "fetched_over_distinct_per_segment": round(fetched / per_segment, 4) if per_segment else None,
            "ms_fetch_only_step": round(t_fetch, 3), "ms_attention_resident": round(t_res, 3),
            "ms_attention_phase_tiered": round(attn_phase_ms, 3),
            "attention_hidden_share": round(hidden, 4) if hidden is not None else None,
            "bytes_offloaded_per_step": off_b,
            "link_gbs_achieved": round(fetched * tb / (step_ms / 1e3) / 1e9, 2),
            "link_both_gbs_achieved": round((fetched * tb + off_b) / (step_ms / 1e3) / 1e9, 2),
            "host_link_gbs_measured": {k: round(v, 2) for k, v in link.items()}}


def e2e_stream_measure(layer, steps, n_slots=2):
    """A single-segment forward step through the C ABI from pinned host buffers,
    streamed: each step's q and segment K/V are copied host -> device on an input
    stream, its route + forward + append run on the compute stream, and its O and
    LSE are copied back on an output stream, over n_slots device slots, so the copies
    of one step overlap the compute of its neighbours (every step still moves all
    of its own bytes, inside the timed region)."""
    import torch
    hga, w = layer.hga, layer.w
    S, T = w.seg_len, w.seg_starts[0]
    p = layer.params(T)
    host_in = [layer.q[T].cpu().pin_memory(), layer.k[:, :, T:T + S].cpu().pin_memory(),
               layer.v[:, :, T:T + S].cpu().pin_memory()]

    class Slot:
        pass

    slots = []
    for n in range(n_slots):
        sl = Slot()
        sl.q = torch.empty_like(layer.q[T])
        sl.k = layer.k if n == 0 else layer.k.clone()
        sl.v = layer.v if n == 0 else layer.v.clone()
        sl.summ = layer.summ if n == 0 else layer.summ.clone()
        sl.idx = torch.empty_like(layer.idx)
        sl.out = torch.empty_like(layer.out)
        sl.lse = torch.empty_like(layer.lse)
        sl.host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (sl.out, sl.lse)]
        sl.in_ready, sl.computed, sl.out_read = (torch.cuda.Event() for _ in range(3))
        slots.append(sl)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in (layer.out, layer.lse))
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()

    def run(n_steps):
        for i in range(n_steps):
            sl = slots[i % n_slots]
            if i >= n_slots:
                s_in.wait_event(sl.computed)  # the slot's previous step has read its inputs
            with torch.cuda.stream(s_in):
                sl.q.copy_(host_in[0], non_blocking=True)
                sl.k[:, :, T:T + S].copy_(host_in[1], non_blocking=True)
                sl.v[:, :, T:T + S].copy_(host_in[2], non_blocking=True)
            sl.in_ready.record(s_in)
            main.wait_event(sl.in_ready)
            if i >= n_slots:
                main.wait_event(sl.out_read)  # the slot's previous step's outputs have left it
            ks, vs = sl.k[:, :, T:], sl.v[:, :, T:]
            hga.hga_route_attn_fwd(p, sl.q, sl.summ, layer.nct, sl.idx, sl.k, sl.v, ks, vs, sl.out, sl.lse)
            hga.hga_build_summaries(sl.k, layer.L, w.batch, w.n_kv_heads, w.head_dim, w.chunk, T // w.chunk,
                                    S // w.chunk, sl.summ, layer.nct)
            sl.computed.record(main)
            s_out.wait_event(sl.computed)
            with torch.cuda.stream(s_out):
                for hbuf, t in zip(sl.host_out, (sl.out, sl.lse)):
                    hbuf.copy_(t, non_blocking=True)
            sl.out_read.record(s_out)
        main.wait_stream(s_out)

    run(4)  # warm-up
    torch.cuda.synchronize()
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record(main)
    s_in.wait_stream(main)
    s_out.wait_stream(main)
    run(steps)
    en.record(main)
    en.synchronize()
    ms = st.elapsed_time(en) / steps
    return {"value": tokens_per_step(w) / (ms / 1000.0), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "scope": f"{steps} steps through the C ABI from pinned host buffers, streamed over {n_slots} device "
                     "slots: "
                     "a step's inputs in and outputs out on their own streams, overlapping the compute of the "
                     "steps next to it"}


def e2e_measure(layer, steps):
    """The whole step through the C ABI from pinned host buffers: every segment's
    inputs (q, segment K/V [, dO]) copied host -> device before its compute and
    its outputs (O, LSE [, dQ, dK, dV]) copied back, all inside the timed region.
    The outputs leave on their own stream from two alternating output sets, so a
    segment's copy-out overlaps the compute of the next."""
    import torch
    w = layer.w
    S = w.seg_len
    host_in = {}
    for T in w.seg_starts:
        host_in[T] = [layer.q[T].cpu().pin_memory(), layer.k[:, :, T:T + S].cpu().pin_memory(),
                      layer.v[:, :, T:T + S].cpu().pin_memory()] + \
                     ([layer.do[T].cpu().pin_memory()] if w.backward else [])
    outs0 = [layer.out, layer.lse] + ([layer.dq, layer.dk, layer.dv] if w.backward else [])
    out_sets = [outs0, [torch.empty_like(t) for t in outs0]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs0] for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]
    s_out = torch.cuda.Stream()
    # the tiered step runs each segment's route and fetches under the attention of the
    # segments before it: its inputs arrive on the route stream, q in a ring of five
    # buffers (the route stream reaches segment s only after the fetches of s - 3, which
    # come after the attention of s - 5)
    # (a pipelined evaluation's route stream runs a segment ahead: a ring of three)
    q_ring = [torch.empty_like(layer.q[w.seg_starts[0]]) for _ in range(5 if w.tiered else
                                                                        3 if layer.pipelined else 1)]
    do_d = torch.empty_like(layer.do[w.seg_starts[0]]) if w.backward else None
    h2d = sum(t.numel() * t.element_size() for ts in host_in.values() for t in ts)
    d2h = sum(t.numel() * t.element_size() for t in outs0) * len(w.seg_starts)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for it in range(steps + 1):
        torch.cuda.synchronize()
        main = torch.cuda.current_stream()
        s.record()
        s_out.wait_stream(main)
        for si, T in enumerate(w.seg_starts):
            hi = host_in[T]
            q_d = q_ring[si % len(q_ring)]
            side_in = w.tiered or layer.pipelined
            if side_in and si == 0:
                layer.route_stream.wait_stream(main)
            with torch.cuda.stream(layer.route_stream if side_in else main):
                q_d.copy_(hi[0], non_blocking=True)
                layer.k[:, :, T:T + S].copy_(hi[1], non_blocking=True)
                layer.v[:, :, T:T + S].copy_(hi[2], non_blocking=True)
                if do_d is not None:
                    do_d.copy_(hi[3], non_blocking=True)
            o = si % 2
            if si >= 2:
                main.wait_event(out_read[o])  # the output set's previous segment has left
            if w.tiered:
                layer.segment_tiered(T, q=q_d, si=si, outs=out_sets[o])
            else:
                layer.segment(T, q=q_d, do=do_d, si=si,
                              outs=out_sets[o] + [None] * (5 - len(out_sets[o])))
            computed[o].record(main)
            s_out.wait_event(computed[o])
            with torch.cuda.stream(s_out):
                for hbuf, t in zip(host_out[o], out_sets[o]):
                    hbuf.copy_(t, non_blocking=True)
            out_read[o].record(s_out)
        if w.tiered:
            layer.end_tiered_step()
        elif layer.pipelined:
            main.wait_stream(layer.route_stream)
        main.wait_stream(s_out)
        e.record()
        e.synchronize()
        if it >= 1:
            times.append(s.elapsed_time(e))
    ms = statistics.mean(times)
    return {"value": tokens_per_step(w) / (ms / 1000.0), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "scope": "every segment of the step through the C ABI from pinned host buffers (outputs copied out "
                     "on their own stream from two alternating output sets)"}


def cpu_procs(args):
    if args.cpu_procs > 0:
        return args.cpu_procs
    return max(1, min(8, cpu_info()["usable_cpus"]))


def run_hga(args, rank, world, local):
    import torch
    from inputs import gen
    import hierarchical_sparse_long_b200 as hga
    from hierarchical_sparse_long_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    hga.lib()
    w = gen.WORKLOADS[args.workload]
    res = measure_layer(w, args, world, local)
    line = {"metric": METRIC, "value": res.pop("value"), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", **res}
    also = list(ALSO_DEFAULT) if (args.also == "auto" and args.workload == "qwen3_16k_fwd") else \
        [a for a in args.also.split(",") if a and a not in ("auto", "none")]
    nested = {}
    for name in also:
        wn = gen.WORKLOADS[name]
        nested[name] = (run_decode_measure(wn, args, world, local) if wn.decode
                        else measure_layer(wn, args, world, local))
    baseline = rank == 0 and world == 1 and not args.no_cpu_baseline
    if baseline:
        import oracle
        oracle.build()
        tok_s, cb = oracle_sample(w, args.cpu_seconds, 1)
        line["cpu_baseline"] = {"value": tok_s, "unit": UNIT, "kind": "oracle", **cb}
        for name, r in nested.items():
            wn = gen.WORKLOADS[name]
            procs = cpu_procs(args) if wn.seq_len > 32768 else 1
            tok_s, cb = oracle_sample(wn, min(args.cpu_seconds, 10.0), procs)
            r["cpu_baseline"] = {"value": tok_s, "unit": UNIT, "kind": "oracle", **cb}
    if nested:
        line["workloads"] = nested
    if rank == 0:
        print(json.dumps(line), flush=True)


class DecodeLayer:
    """Device state of a decode step: the sequences' K/V (history and local window
    in one buffer per head), the history's chunk summaries and each sequence's new
    token (the last of its local window)."""

    def __init__(self, w):
        import torch
        from inputs import gen
        import hierarchical_sparse_long_b200 as hga
        self.w, self.hga, self.torch = w, hga, torch
        dev = torch.device("cuda")
        self.T, self.n_local, self.Ltot = w.seg_starts[0], w.seg_len, w.seq_len
        self.k = gen.keys_torch(w, 0, self.Ltot, dev).contiguous()
        self.v = gen.values_torch(w, 0, self.Ltot, dev).contiguous()
        self.q = gen.queries_torch(w, self.Ltot - 1, self.Ltot, dev).contiguous()  # [B][Hq][1][D]
        self.nc = self.T // w.chunk
        self.summ = torch.zeros(w.batch, w.n_kv_heads, self.nc, w.head_dim, device=dev)
        hga.hga_build_summaries(self.k, self.Ltot, w.batch, w.n_kv_heads, w.head_dim, w.chunk, 0, self.nc,
                                self.summ, self.nc)
        self.p = hga.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                            topk=w.topk, seg_len=1, n_hist_chunks=self.nc, dtype=hga.HGA_BF16,
                            hist_head_stride=self.Ltot, seg_head_stride=self.Ltot, chunk=w.chunk, q_block=1,
                            sink_chunks=w.sink_chunks)
        self.idx = torch.empty(w.batch, w.n_kv_heads, 1, w.topk, device=dev, dtype=torch.int32)
        self.out = torch.empty(w.batch, w.n_q_heads, 1, w.head_dim, device=dev, dtype=torch.bfloat16)
        self.lse = torch.empty(w.batch, w.n_q_heads, 1, device=dev)
        self.ws = torch.empty(hga.hga_attn_decode_workspace_size(self.p, self.n_local) // 4 + 64, device=dev)
        torch.cuda.synchronize()

    def step(self, ev=None, q=None):
        rec = ev.record if ev is not None else (lambda name: None)
        q = self.q if q is None else q
        T = self.T
        rec("route")
        self.hga.hga_route(self.p, q, self.summ, self.nc, self.idx)
        rec("attn_decode")
        self.hga.hga_attn_decode(self.p, q, self.k, self.v, self.k[:, :, T:], self.v[:, :, T:], self.n_local,
                                 self.idx, self.out, self.lse, self.ws)
        rec(None)
        return 3


def run_decode_measure(w, args, world, local):
    """Times a decode workload: one step = route + decode attention of one new token
    per sequence (query tok/s = tokens generated per second); returns its JSON fields."""
    import torch
    import hierarchical_sparse_long_b200 as hga
    layer = DecodeLayer(w)
    flush = torch.empty(256 * 1024 * 1024 // 4, device="cuda", dtype=torch.float32)
    for _ in range(args.warmup):
        flush_l2(flush)
        layer.step()
    torch.cuda.synchronize()
    if hga.hga_get_device_status() != 0:
        raise RuntimeError("device status reported an error during warm-up")
    # the timed graph has no event nodes inside; a second graph of the same step with
    # events between its calls gives the per-kernel times, replayed afterwards
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        graph_launches = layer.step()
    gev = PhaseEvents(external=True)
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph):
        layer.step(ev=gev)
    for gr in (graph, pgraph):
        flush_l2(flush)
        gr.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    phases, launches = [], 0
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for s_ in range(args.steps):
        flush_l2(flush)
        starts[s_].record()
        graph.replay()
        ends[s_].record()
        launches += graph_launches
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(starts, ends)), world, "cuda")
    value = job_throughput(tokens_per_step(w), args.steps, world, total_ms)
    for s_ in range(args.steps):
        flush_l2(flush)
        pgraph.replay()
        torch.cuda.synchronize()
        phases.append(gev.totals())
    status = hga.hga_get_device_status()
    ph = {}
    for ev in phases:
        for k, v in ev.items():
            ph[k] = ph.get(k, 0.0) + v
    peaks, peak_src = measured_peaks()
    B, Hq, Hkv, D = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    keff = min(w.topk, layer.nc)
    route_b = B * Hkv * layer.nc * D * 4 + B * Hq * D * 2 + B * Hkv * w.topk * 4
    dec_b = B * Hkv * (keff * w.chunk + layer.n_local) * D * 2 * 2 + 2 * B * Hq * D * 2 + B * Hkv * w.topk * 4
    kernels = {
        "route": {"bound": "hbm", "ms_per_launch": ph["route"] / args.steps,
                  "achieved": route_b * args.steps / (ph["route"] / 1e3) / 1e9, "unit": "GB/s"},
        "attn_decode": {"bound": "hbm", "ms_per_launch": ph["attn_decode"] / args.steps,
                        "achieved": dec_b * args.steps / (ph["attn_decode"] / 1e3) / 1e9, "unit": "GB/s"},
    }
    for k, v in kernels.items():
        v["frac"] = round(v["achieved"] / peaks["hbm_gbs"], 4)
        v["achieved"] = round(v["achieved"], 2)
        v["ms_per_launch"] = round(v["ms_per_launch"], 4)
    kd = kernels["attn_decode"]
    roof = {"bound": "hbm", "kernel": "hga_attn_decode", "achieved": kd["achieved"], "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": kd["frac"], "traffic": kernel_traffic("attn_decode", w.name),
            "peak_source": f"{peak_src}: MEASURED_PEAKS.json hbm_gbs",
            "units_per_launch": "K and V of the routed chunks and the local window once per (sequence, kv head), "
                                "plus q, O and the route table"}
    res = {"value": value, "unit": UNIT, "ms_per_step": total_ms / args.steps,
           "config": {**workload_config(w, world),
                      "l2": "flushed before every timed step (256 MiB write)",
                      "launch": "one CUDA graph replay per step",
                      "kernel_times": "from as many replays of the same step with CUDA events between its "
                                      "library calls, after the timed region"},
           "roofline": roof, "kernels": kernels, "clocks": clocks, "gpu_launches": launches,
           "device_status": status}
    res["e2e"] = decode_e2e(layer, max(2, min(args.steps, 5)))
    del layer, graph
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_decode(args, rank, world, local):
    """bench.py with a decode workload as the headline."""
    import torch
    from inputs import gen
    import hierarchical_sparse_long_b200 as hga
    from hierarchical_sparse_long_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    hga.lib()
    w = gen.WORKLOADS[args.workload]
    res = run_decode_measure(w, args, world, local)
    line = {"metric": METRIC, "value": res.pop("value"), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", **res}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        tok_s, cb = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tok_s, "unit": UNIT, "kind": "oracle", **cb}
    if rank == 0:
        print(json.dumps(line), flush=True)


def decode_e2e(layer, steps):
    """The decode step through the C ABI from pinned host buffers: the new tokens' q, k
    and v copied in (k / v into the last slot of each local window), route and decode,
    O and LSE copied back, all inside the timed region."""
    import torch
    w, T, Lt = layer.w, layer.T, layer.Ltot
    host_q = layer.q.cpu().pin_memory()
    host_k = layer.k[:, :, Lt - 1:Lt].cpu().pin_memory()
    host_v = layer.v[:, :, Lt - 1:Lt].cpu().pin_memory()
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (layer.out, layer.lse)]
    q_d = torch.empty_like(layer.q)
    h2d = sum(t.numel() * t.element_size() for t in (host_q, host_k, host_v))
    d2h = sum(t.numel() * t.element_size() for t in (layer.out, layer.lse))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for it in range(steps + 1):
        torch.cuda.synchronize()
        s.record()
        q_d.copy_(host_q, non_blocking=True)
        layer.k[:, :, Lt - 1:Lt].copy_(host_k, non_blocking=True)
        layer.v[:, :, Lt - 1:Lt].copy_(host_v, non_blocking=True)
        layer.step(q=q_d)
        host_out[0].copy_(layer.out, non_blocking=True)
        host_out[1].copy_(layer.lse, non_blocking=True)
        e.record()
        e.synchronize()
        if it >= 1:
            times.append(s.elapsed_time(e))
    ms = statistics.mean(times)
    return {"value": tokens_per_step(w) / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "scope": "the decode step through the C ABI from pinned host buffers"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args, int(os.environ.get("RANK", "0")))
        return
    rank, world, local = dist_setup()
    from inputs import gen
    try:
        if gen.WORKLOADS[args.workload].decode:
            run_decode(args, rank, world, local)
        else:
            run_hga(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
