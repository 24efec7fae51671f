#!/usr/bin/env python
"""Benchmark of the HGA attention layer on B200.

Default workload: the Qwen3-8B-shaped layer at 16K context (32 query heads,
8 KV heads, head_dim 128, bf16, 14,336 detached history tokens + a 2,048-token
active segment, chunk 64, query block 64, top-16 chunks).  One step is the
layer's hot path over that segment: route the 32 query blocks, exact-token
attention forward over the routed chunks + the causal segment, and the
detach-time summary append of the segment's 32 chunks (with --workload
qwen3_16k_train the step also runs the backward; qwen3_128k_eval runs the
32 segments of a 131,072-token evaluation as one step).

Metric: query tokens/s (active query tokens processed per second, all heads).
Inputs are seeded synthetic tensors (inputs/gen.py) with the workload's
shapes and key-offset structure; the L2 is flushed before every timed step.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HGA attn query tok/s at 16K & 128K ctx; % of HBM / tensor-pipe roofline"
UNIT = "query tok/s"
KERNEL_SOURCES = {"attn_fwd": ["hierarchical_sparse_long_b200/csrc/attn_fwd_tc.cu",
                               "hierarchical_sparse_long_b200/csrc/attn_simt.cu",
                               "hierarchical_sparse_long_b200/csrc/tc_ptx.cuh"]}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--workload", default="qwen3_16k_fwd",
                    choices=["qwen3_16k_fwd", "qwen3_16k_train", "qwen3_128k_eval"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def dist_setup(n_gpus):
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


def file_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        fp = os.path.join(ROOT, p)
        if os.path.exists(fp):
            h.update(open(fp, "rb").read())
    return h.hexdigest()[:16]


def measured_peaks():
    fp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(fp):
        d = json.load(open(fp))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(kernel):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel source is unchanged since."""
    fp = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(fp):
        return None
    d = json.load(open(fp)).get(kernel)
    if not d or d.get("source_hash") != file_hash(KERNEL_SOURCES.get(kernel, [])):
        return None
    return d.get("bytes_per_launch")


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
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ workload state
class Layer:
    """Device state of one HGA layer: K/V of the whole sequence in one buffer per
    head, resident chunk summaries, the active segment's queries."""

    def __init__(self, w, seed_offset=0):
        import numpy as np
        import torch

        from inputs import gen
        import hierarchical_sparse_long_b200 as hga
        self.w, self.hga, self.torch = w, hga, torch
        L = w.seq_len
        self.L = L
        dt = torch.bfloat16
        t0 = time.time()
        self.k_host = torch.from_numpy(gen.keys(w, 0, L)).to(dt).pin_memory()
        self.v_host = torch.from_numpy(gen.values(w, 0, L)).to(dt).pin_memory()
        self.k = self.k_host.cuda()
        self.v = self.v_host.cuda()
        # queries of every processed segment
        self.q_host = {}
        self.q = {}
        self.do = {}
        self.do_host = {}
        for T in w.seg_starts:
            qh = torch.from_numpy(gen.queries(w, T, T + w.seg_len)).to(dt).pin_memory()
            self.q_host[T] = qh
            self.q[T] = qh.cuda()
            if w.backward:
                dh = torch.from_numpy(gen.grad_out(w, T, T + w.seg_len)).to(dt).pin_memory()
                self.do_host[T] = dh
                self.do[T] = dh.cuda()
        self.gen_seconds = time.time() - t0
        self.nct = L // w.chunk
        self.summ = torch.zeros(w.batch, w.n_kv_heads, self.nct, w.head_dim, device="cuda")
        nqb = w.seg_len // w.q_block
        self.idx = torch.empty(w.batch, w.n_kv_heads, nqb, w.topk, device="cuda", dtype=torch.int32)
        self.out = torch.empty(w.batch, w.n_q_heads, w.seg_len, w.head_dim, device="cuda", dtype=dt)
        self.lse = torch.empty(w.batch, w.n_q_heads, w.seg_len, device="cuda")
        if w.backward:
            self.dq = torch.empty(self.out.shape, device="cuda", dtype=torch.float32)
            self.dk = torch.empty(w.batch, w.n_kv_heads, w.seg_len, w.head_dim, device="cuda", dtype=torch.float32)
            self.dv = torch.empty_like(self.dk)
            p = self.params(w.seg_starts[-1])
            self.ws = torch.empty(hga.hga_attn_bwd_workspace_size(p) // 4 + 64, device="cuda")
        # history that exists before the first timed segment is summarised once
        first = w.seg_starts[0] // w.chunk
        if first:
            hga.hga_build_summaries(self.k, L, w.batch, w.n_kv_heads, w.head_dim, w.chunk, 0, first, self.summ,
                                    self.nct)
        torch.cuda.synchronize()

    def params(self, T, **kw):
        w = self.w
        p = self.hga.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                            topk=w.topk, seg_len=w.seg_len, n_hist_chunks=T // w.chunk, dtype=self.hga.HGA_BF16,
                            hist_head_stride=self.L, seg_head_stride=self.L, chunk=w.chunk, q_block=w.q_block)
        for k, v in kw.items():
            setattr(p, k, v)
        return p

    def segment(self, T, ev=None, q=None, do=None):
        """One segment of the hot path; returns the number of library kernels launched."""
        hga, w = self.hga, self.w
        p = self.params(T)
        q = self.q[T] if q is None else q
        ks = self.k[:, :, T:]
        vs = self.v[:, :, T:]
        hga.hga_route(p, q, self.summ, self.nct, self.idx)
        if ev is not None:
            ev[0].record()
        hga.hga_attn_fwd(p, q, self.k, self.v, ks, vs, self.idx, self.out, self.lse)
        if ev is not None:
            ev[1].record()
        launches = 2
        if w.backward:
            hga.hga_attn_bwd(p, q, self.k, self.v, ks, vs, self.idx, self.out, self.lse,
                             self.do[T] if do is None else do, self.dq, self.dk, self.dv, self.ws)
            launches += 3
        # detach: the segment's chunks become routable history
        hga.hga_build_summaries(self.k, self.L, w.batch, w.n_kv_heads, w.head_dim, w.chunk, T // w.chunk,
                                w.seg_len // w.chunk, self.summ, self.nct)
        return launches + 1

    def step(self, ev=None):
        n = 0
        for i, T in enumerate(self.w.seg_starts):
            n += self.segment(T, ev=ev if i == len(self.w.seg_starts) - 1 else None)
        return n


def attn_flops(w, T):
    """Algorithmic FLOPs of one forward launch: 4*D*(k_eff*c + i + 1) per query row per head."""
    keff = min(w.topk, T // w.chunk)
    S = w.seg_len
    per_head = 4 * w.head_dim * (keff * w.chunk * S + S * (S + 1) / 2)
    return per_head * w.batch * w.n_q_heads


def flush_l2(buf):
    buf.add_(1)


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(w, target_seconds, rank0=True):
    """Times the CPU oracle on a bounded sample of the workload; returns (tok/s, desc, cores)."""
    import numpy as np

    import oracle
    from inputs import gen
    T = w.seg_starts[-1]
    S, D = w.seg_len, w.head_dim
    q = gen.queries(w, T, T + S)
    k_all = gen.keys(w, 0, T + S)
    v_all = gen.values(w, 0, T + S)
    sh = oracle.shape(w.batch, w.n_q_heads, w.n_kv_heads, D, w.chunk, w.q_block, w.topk, S, T // w.chunk)
    t0 = time.perf_counter()
    summ_new = oracle.summaries(k_all[:, :, T:], w.chunk)  # detach-time summaries of the segment
    summ = oracle.summaries(k_all[:, :, :T], w.chunk) if T else np.zeros((w.batch, w.n_kv_heads, 0, D))
    t_summ = time.perf_counter() - t0
    t0 = time.perf_counter()
    idx, _, _ = oracle.route(sh, q, summ)
    t_route = time.perf_counter() - t0
    # attention rows: whole query blocks (all heads), latest blocks first, until the budget is spent
    nqb = S // w.q_block
    rows_done, t_attn, blocks = 0, 0.0, []
    for m in list(range(nqb - 1, -1, -max(1, nqb // 8))):
        rows = np.array([(b * w.n_q_heads + h) * S + m * w.q_block + i for b in range(w.batch)
                         for h in range(w.n_q_heads) for i in range(w.q_block)], dtype=np.int64)
        t0 = time.perf_counter()
        oracle.attn_fwd(sh, q, k_all[:, :, :T], v_all[:, :, :T], k_all[:, :, T:], v_all[:, :, T:], idx, rows=rows)
        t_attn += time.perf_counter() - t0
        blocks.append(m)
        if t_attn + t_route > target_seconds:
            break
    # per-token cost: attention of the sampled blocks, scaled to the segment's block mix by the
    # attended-key count, plus the whole-segment route and summary work
    keff = min(w.topk, T // w.chunk)
    cost = lambda m: keff * w.chunk + m * w.q_block + (w.q_block + 1) / 2  # mean keys per row of block m
    frac = sum(cost(m) for m in blocks) / sum(cost(m) for m in range(nqb))
    seg_seconds = t_attn / frac + t_route + t_summ
    tok_s = S * w.batch / seg_seconds
    desc = (f"oracle fp64 single-thread: summaries + route of one {S}-token segment at T={T}, attention of "
            f"query blocks {sorted(blocks)} (all {w.n_q_heads} heads) scaled by attended-key count to the "
            f"segment; {t_attn + t_route + t_summ:.1f} s CPU")
    return tok_s, desc, 1


# ------------------------------------------------------------------ arms
def run_reference(args, rank, world):
    from inputs import gen
    if rank != 0:
        return
    w = gen.WORKLOADS[args.workload]
    import oracle
    oracle.build()
    per_step = []
    desc = ""
    budget = max(2.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for s in range(args.warmup + args.steps):
        tok_s, desc, cores = oracle_sample(w, budget)
        if s >= args.warmup:
            per_step.append(tok_s)
    v = statistics.median(per_step)
    ms = w.seg_len * w.batch / v * 1000 * len(w.seg_starts)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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
    layer = Layer(w)
    flush = torch.empty(256 * 1024 * 1024 // 4, device="cuda", dtype=torch.float32)
    ev_attn = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for _ in range(args.warmup):
        flush_l2(flush)
        layer.step()
    torch.cuda.synchronize()
    if hga.hga_get_device_status() != 0:
        raise RuntimeError("device status reported an error during warm-up")
    sampler = ClockSampler(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    attn_ms = []
    launches = 0
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for s in range(args.steps):
        flush_l2(flush)
        starts[s].record()
        launches += layer.step(ev=ev_attn)
        ends[s].record()
        ends[s].synchronize()
        attn_ms.append(ev_attn[0].elapsed_time(ev_attn[1]))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    tokens_per_step = w.seg_len * w.batch * len(w.seg_starts)
    value = tokens_per_step * args.steps * world / (total_ms / 1000.0)
    status = hga.hga_get_device_status()

    # end to end through the C ABI from pinned host buffers: H2D of the step's
    # inputs (active-segment q, k, v [and dO]), D2H of the outputs
    e2e = e2e_measure(layer, max(3, min(args.steps, 10)))

    peaks, peak_src = measured_peaks()
    T_last = w.seg_starts[-1]
    fl = attn_flops(w, T_last)
    a_ms = statistics.mean(attn_ms)
    achieved = fl / (a_ms / 1000.0) / 1e12
    peak = peaks["bf16_tflops"]
    roof = {"bound": "tensor", "kernel": "hga_attn_fwd", "achieved": round(achieved, 2), "peak": peak,
            "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": kernel_traffic("attn_fwd"),
            "peak_source": peak_src + " (burst bf16)", "algorithmic_flops_per_launch": fl,
            "launch_ms": round(a_ms, 4)}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                       "head_dim": w.head_dim, "context": w.seq_len, "seg_len": w.seg_len, "topk": w.topk,
                       "chunk": w.chunk, "q_block": w.q_block, "segments_per_step": len(w.seg_starts),
                       "backward": w.backward, "parallelism": f"replicas x{world}",
                       "l2": "flushed before every timed step (256 MiB write)"},
            "roofline": roof, "clocks": clocks, "gpu_launches": launches, "e2e": e2e,
            "device_status": status}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, desc, cores = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tok_s, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)


def e2e_measure(layer, steps):
    import torch
    w = layer.w
    T = w.seg_starts[-1]
    qh = layer.q_host[T]
    kh = layer.k_host[:, :, T:].contiguous().pin_memory()
    vh = layer.v_host[:, :, T:].contiguous().pin_memory()
    doh = layer.do_host.get(T)
    out_h = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
    lse_h = torch.empty(layer.lse.shape, dtype=layer.lse.dtype).pin_memory()
    grads_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (layer.dq, layer.dk, layer.dv)] \
        if w.backward else []
    q_d = torch.empty_like(layer.q[T])
    do_d = torch.empty_like(layer.do[T]) if doh is not None else None
    h2d = qh.numel() * 2 + kh.numel() * 2 + vh.numel() * 2 + (doh.numel() * 2 if doh is not None else 0)
    d2h = out_h.numel() * 2 + lse_h.numel() * 4
    if w.backward:
        d2h += layer.dq.numel() * 4 + layer.dk.numel() * 4 + layer.dv.numel() * 4
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for it in range(steps + 2):
        torch.cuda.synchronize()
        s.record()
        q_d.copy_(qh, non_blocking=True)
        layer.k[:, :, T:].copy_(kh, non_blocking=True)
        layer.v[:, :, T:].copy_(vh, non_blocking=True)
        if do_d is not None:
            do_d.copy_(doh, non_blocking=True)
        layer.segment(T, q=q_d, do=do_d)
        out_h.copy_(layer.out, non_blocking=True)
        lse_h.copy_(layer.lse, non_blocking=True)
        for hbuf, t in zip(grads_h, (layer.dq, layer.dk, layer.dv) if w.backward else ()):
            hbuf.copy_(t, non_blocking=True)
        e.record()
        e.synchronize()
        if it >= 2:
            times.append(s.elapsed_time(e))
    ms = statistics.mean(times)
    return {"value": w.seg_len * w.batch / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "scope": "last segment of the workload through the C ABI from pinned host buffers"}


def main():
    args = parse()
    rank, world, local = (0, 1, 0)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_hga(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
