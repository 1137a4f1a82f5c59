#!/usr/bin/env python
"""Benchmark of one Light Forcing HSA attention call on B200.

A step is one whole HSA call on resident inputs: block/frame mean pooling, the
two-level selection (frames, then blocks, in one launch) and block-sparse
attention (three kernels of liblf_hsa.so, called through the C ABI, plus the
merge kernel when the attention splits the lists of the tail). The default workload is the
480p-shaped layer call (batch 1, 12 heads, head_dim 128, 1560-token frames,
21 KV frames = sink + 16 memory + recent + 3-frame current chunk, frame top-4,
block top-k for 80 % block sparsity), drawn by ``lf_synth``.

Metric: effective TFLOP/s on kept blocks = (4 * valid query rows * valid kept
key tokens * head_dim, summed over every query block) / time of the whole call.
The line also carries the microseconds of every kernel, the pooling and
selection bandwidth, the attention kernel's roofline fraction, the oracle's CPU
throughput on a bounded sample, and an end-to-end number with host buffers.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run; each rank runs the same call on
its own GPU (the call shards by (batch, head) with no exchange: weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSA µs/call and effective TFLOPS on kept blocks (% bf16 peak); select GB/s"
L2_FLUSH_BYTES = 512 << 20
E2E_GROUPS = 4  # head groups of the pipelined end-to-end measurement


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="layer480p")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-budget-s", type=float, default=15.0)
    p.add_argument("--no-configs", action="store_true",
                   help="skip the per-config report (all five workloads, rollout per chunk)")
    p.add_argument("--config-steps", type=int, default=30)
    p.add_argument("--only-report", choices=["layer480p_1d", "layer480p_fp8", "longvideo480p_ivf", "cached_pooled_keys"],
                   default=None,
                   help="run only this extra report after the main line (skips the other configs); "
                        "used to profile one of its kernels")
    p.add_argument("--strong", action="store_true",
                   help="N > 1: split one call's (batch, head) units across the ranks (strong scaling); "
                        "default: each rank takes a whole workload's units of a call whose batch grows "
                        "with N (weak scaling)")
    return p.parse_args()


def _workload(name):
    import lf_synth
    return lf_synth.CONFIGS[name]


def _kb(L, shape, w):
    if w.topk_blocks:
        return w.topk_blocks
    n_sel = L.lf_frames_selected(shape, w.chunk_index, w.topk_frames)
    return L.lf_blocks_for_sparsity(w.sparsity, shape.Nkv, n_sel, shape.bpf)


def credited_flops(block_list, block_count, F, bpf, D, n_cur):
    """4 * valid queries * valid kept keys * D over every query block (host, numpy)."""
    import numpy as np
    lst = block_list.reshape(-1, block_list.shape[-1])
    cnt = block_count.reshape(-1)
    Rq = n_cur * bpf
    rem = F - 64 * (bpf - 1)
    total = 0
    for row in range(cnt.size):
        r = row % Rq
        q_valid = rem if (r % bpf) == bpf - 1 else 64
        ids = lst[row, :cnt[row]]
        kv_valid = int(np.where((ids % bpf) == bpf - 1, rem, 64).sum())
        total += 4 * q_valid * kv_valid * D
    return float(total)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                clk, cmax, pw = float(parts[0]), float(parts[1]), float(parts[2])
            except ValueError:
                continue
            mx = cmax
            if pw > 200.0:  # under load
                sm.append(clk)
                for n, flag in zip(names, parts[4:8]):
                    if flag.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples_under_load": len(sm)}


def _dist():
    """(dist module or None, rank, world size, local rank). One process per GPU;
    the process group (NCCL, or gloo when LF_DIST_BACKEND=gloo for host-only
    tests) carries only the barrier and the max-over-ranks timing."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group(os.environ.get("LF_DIST_BACKEND", "nccl"), timeout=timedelta(seconds=120))
        return dist, dist.get_rank(), ws, int(os.environ.get("LOCAL_RANK", "0"))
    return None, 0, 1, 0


def _reduce_over_ranks(dist, x, op="max"):
    if dist is None:
        return x
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def _max_over_ranks(dist, x):
    return _reduce_over_ranks(dist, x, "max")


def _idle_rank(a, dist, ws):
    """A rank with no (batch, head) units (strong scaling with more ranks than
    units): it takes the same collective steps as a working rank, in the same order."""
    if dist is None:
        return
    dist.barrier()                       # before the timed region
    dist.barrier()                       # after it
    _reduce_over_ranks(dist, 0.0, "max")  # step time
    _reduce_over_ranks(dist, 0.0, "sum")  # credited FLOPs
    _reduce_over_ranks(dist, 0.0, "max")  # end-to-end time
    dist.barrier()
    dist.destroy_process_group()


def _rank_workload(name, rank):
    """Weak scaling: the call's batch grows with the number of ranks and rank i
    takes the contiguous (batch, head) units [i*U, (i+1)*U), U = one workload's
    batch*heads (shard_units of the grown call); its slice is drawn directly
    (the workload's generator with the seed offset by the rank)."""
    import lf_synth
    w = lf_synth.CONFIGS[name]
    return w if rank == 0 else lf_synth.workload(name, seed=w.seed + 1000 * rank)


def _rank_inputs(L, lf_synth, name, rank, ws, strong):
    """(workload, per-rank LfShape or None, q, k, v on the host, unit range).
    strong: one call of the workload, its (batch, head) units split across the
    ranks (shard_shape); otherwise every rank takes a whole workload's units of a
    call whose batch grows with the ranks."""
    if strong and ws > 1:
        w = lf_synth.CONFIGS[name]
        q, k, v = lf_synth.make_qkv(w)
        full = L.shape_from_workload(w)
        shape, u0, u1 = L.shard_shape(full, ws, rank)
        if shape is None:
            return w, None, None, None, None, (u0, u1)
        q, k, v = (L.unit_view(t, u0, u1).contiguous() for t in (q, k, v))
        return w, shape, q, k, v, (u0, u1)
    w = _rank_workload(name, rank)
    U = w.batch * w.heads
    q, k, v = lf_synth.make_qkv(w)
    return w, L.shape_from_workload(w), q, k, v, (rank * U, (rank + 1) * U)


def _oracle_sample(w, budget_s, q, k, v, block_list=None, block_count=None):
    """Time the fp64 oracle on a bounded sample of the call; returns a dict with
    the extrapolated seconds per call and the credited FLOPs of the call."""
    import numpy as np
    import oracle
    s = oracle.shape_of(w)
    t0 = time.perf_counter()
    qp, kp, kf = oracle.pool(s, q, k)
    t_pool = time.perf_counter() - t0
    t0 = time.perf_counter()
    sel, _ = oracle.select_frames(s, w.chunk_index, w.topk_frames, qp, kf)
    n_sel = sel.shape[-1]
    kb = w.topk_blocks or oracle.blocks_for_sparsity(w.sparsity, s.Nkv, n_sel, s.bpf)
    lst, cnt, _ = oracle.select_blocks(s, w.chunk_index, kb, qp, kp, sel)
    t_sel = time.perf_counter() - t0
    total_rows = s.batch * s.heads * s.Lq
    rng = np.random.default_rng(0)
    # grow the attention sample until the budget is spent
    rows_done, t_att, n = 0, 0.0, 64
    while t_att < max(0.5, budget_s - t_pool - t_sel) and rows_done < total_rows:
        rows = rng.integers(0, total_rows, size=n)
        t0 = time.perf_counter()
        oracle.attention(s, q, k, v, lst, cnt, rows=rows)
        t_att += time.perf_counter() - t0
        rows_done += n
        n = min(n * 2, 4096)
    t_call = t_pool + t_sel + t_att * total_rows / rows_done
    flops = credited_flops(lst, cnt, s.frame_tokens, s.bpf, s.head_dim, s.n_cur)
    cpu = platform.processor() or platform.machine()
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    cpu = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    sample = (f"fp64 oracle, 1 thread on {cpu} (nproc {os.cpu_count()}): full pooling "
              f"({t_pool:.2f} s) and selection ({t_sel:.2f} s), attention on {rows_done} of "
              f"{total_rows} query rows ({t_att:.2f} s) extrapolated linearly to the whole call")
    return dict(t_call=t_call, flops=flops, sample=sample, wall=t_pool + t_sel + t_att)


def run_reference(a):
    """The oracle as the reference arm: same metric, config and unit."""
    dist, rank, ws, _ = _dist()
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    import lf_synth
    w = _workload(a.workload)
    q, k, v = lf_synth.make_qkv(w)
    n_steps = a.steps + a.warmup
    per_step = max(2.0, 150.0 / max(1, n_steps))
    times = []
    last = None
    for i in range(n_steps):
        r = _oracle_sample(w, per_step, q, k, v)
        if i >= a.warmup:
            times.append(r["t_call"])
        last = r
    t = statistics.mean(times) if times else last["t_call"]
    value = last["flops"] / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (lf_synth, seeded; stands in for the pages' VBench 480p rollouts)",
        "config": _config(w, None),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def _config(w, kb):
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "head_dim": w.head_dim,
            "frame_tokens": w.frame_tokens, "kv_frames": w.n_frames,
            "frames": {"sink": w.n_sink, "memory": w.n_mem, "recent": w.n_recent,
                       "current": w.n_cur},
            "q_tokens": w.q_tokens, "kv_tokens": w.kv_tokens, "block_tokens": w.block_tokens,
            "topk_frames": w.topk_frames, "topk_blocks": kb, "target_sparsity": w.sparsity,
            "chunk_index": w.chunk_index, "l2": "flushed before every step (512 MiB write)"}


def _attn_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if the
    kernel source has not changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "attn_layer480p_ncu.json")
    src = os.path.join(ROOT, "block_sparse_attention_lf_b200", "csrc", "lf_attn.cu")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return d.get("dram_bytes_per_launch") if d.get("kernel_src_sha256") == sha else None


def _pct(xs, p):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, max(0, int(round(p / 100.0 * (len(xs) - 1)))))]


def measure_call(L, shape, chunk_index, topk_frames, kb, q, k, v, steps, warmup, flush, cached=False):
    """Time the calls of one HSA call on resident inputs (L2 flushed before every
    step): the whole call with no events between its kernels, and each kernel in a
    second pass with events between them; returns µs (mean, p10, p90), credited
    FLOPs and pooling bytes. ``cached``: pooled keys of the past frames persist from a
    first full pooling, and each call re-pools only the current chunk's frames
    and the queries (lf_pool_range)."""
    import torch
    call = L.HSACall(shape, chunk_index, topk_frames, kb)
    nf, nc = shape.n_frames, shape.n_cur

    def pool():
        b_ = call.buf
        if cached:
            L.lf_pool_range(shape, q, k, nf - nc, nf, b_.q_pool, b_.k_pool, b_.k_frame)
        else:
            call.pool(q, k)
    b = call.buf
    stream = torch.cuda.current_stream()
    for _ in range(max(3, warmup)):
        call(q, k, v)
    torch.cuda.synchronize()
    flops = credited_flops(b.block_list.cpu().numpy(), b.block_count.cpu().numpy(),
                           shape.frame_tokens, shape.bpf, shape.head_dim, shape.n_cur)
    E = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        e = E[i]
        e[0].record(stream)
        pool()
        e[1].record(stream)
        call.select()
        e[2].record(stream)
        e[3].record(stream)
        call.attend(q, k, v)
        e[4].record(stream)
    # the whole call, with no events between its kernels (they would stop the programmatic
    # dependent launches)
    EC = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        EC[i][0].record(stream)
        pool()
        call.select()
        call.attend(q, k, v)
        EC[i][1].record(stream)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    if st != 0:
        raise SystemExit(f"device error: {st} {detail:#x}")

    def us(i0, i1):
        xs = [E[j][i0].elapsed_time(E[j][i1]) * 1e3 for j in range(steps)]
        return statistics.mean(xs), _pct(xs, 10), _pct(xs, 90)

    xc = [e0.elapsed_time(e1) * 1e3 for e0, e1 in EC]
    total = (statistics.mean(xc), _pct(xc, 10), _pct(xc, 90))

    pool_bytes = (q.numel() + k.numel()) * 2 + (b.q_pool.numel() + b.k_pool.numel() + b.k_frame.numel()) * 4
    if cached:
        kf = k.numel() * nc // nf
        pool_bytes = (q.numel() + kf) * 2 + (b.q_pool.numel() + (b.k_pool.numel() + b.k_frame.numel()) * nc // nf) * 4
    return dict(pool=us(0, 1), select=us(1, 2), attn=us(3, 4),
                total=total, flops=flops, pool_bytes=pool_bytes, kb=kb,
                list_entries=int(b.block_count.sum().item()))


def _summary(m, peaks):
    t = m["total"][0]
    att = m["attn"][0]
    return {
        "us_per_call": round(t, 2), "us_p10_p90": [round(m["total"][1], 2), round(m["total"][2], 2)],
        "kernels_us": {k: round(m[k][0], 2) for k in ("pool", "select", "attn")},
        "kept_tflop": round(m["flops"] / 1e12, 5), "topk_blocks": m["kb"],
        "tflops_call": round(m["flops"] / (t * 1e-6) / 1e12, 1),
        "attn_tflops": round(m["flops"] / (att * 1e-6) / 1e12, 1),
        "attn_frac_of_bf16_peak": round(m["flops"] / (att * 1e-6) / 1e12 / peaks["bf16"], 4),
        "pool_frac_of_hbm": round(m["pool_bytes"] / (m["pool"][0] * 1e-6) / 1e9 / peaks["hbm"], 3),
        "select_over_attn": round((m["pool"][0] + m["select"][0]) / att, 4),
    }


def config_report(L, lf_synth, peaks, steps, flush):
    """The other workloads of the benchmark plan at one GPU: tiny, long-video,
    pattern-diversity batch at two sparsities, and the 7-chunk rollout with the
    Chunk-Aware Growth budgets (per chunk and the total)."""
    import torch
    out = {}
    for name, kbs in (("tiny", [None]), ("longvideo480p", [None]), ("patterns480p", [12, 6])):
        w = lf_synth.CONFIGS[name]
        shape = L.shape_from_workload(w)
        q, k, v = (t.cuda() for t in lf_synth.make_qkv(w))
        for kb in kbs:
            kbv = kb or _kb(L, shape, w)
            m = measure_call(L, shape, w.chunk_index, w.topk_frames, kbv, q, k, v, steps, 3, flush)
            out[name if kb is None else f"{name}_kb{kb}"] = _summary(m, peaks)
        del q, k, v
        torch.cuda.empty_cache()
    w = lf_synth.CONFIGS["rollout480p"]
    qa, ka, va = lf_synth.make_rollout_qkv(w)
    n = int(w.extra["n_chunks"])
    st, s_out, beta = L.lf_cag_budget(list(range(1, n + 1)), list(range(1, n + 1)), w.extra["s_base"], w.sparsity)
    if st != 0:
        raise SystemExit(f"CAG budgets infeasible: status {st}")
    chunks, tot_us, tot_flops = [], 0.0, 0.0
    for c in range(1, n + 1):
        wc, q, k, v = lf_synth.rollout_chunk(w, qa, ka, va, c)
        shape = L.shape_from_workload(wc)
        n_sel = L.lf_frames_selected(shape, c, wc.topk_frames)
        kb = shape.bpf if c == 1 else L.lf_blocks_for_sparsity(s_out[c - 1], shape.Nkv, n_sel, shape.bpf)
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        m = measure_call(L, shape, c, wc.topk_frames, kb, q, k, v, steps, 3, flush)
        sm = _summary(m, peaks)
        sm["chunk"], sm["s_i"] = c, round(float(s_out[c - 1]), 6)
        chunks.append(sm)
        tot_us += m["total"][0]
        tot_flops += m["flops"]
    out["rollout480p"] = {"beta": round(float(beta), 6), "chunks": chunks, "total_us": round(tot_us, 1),
                          "tflops": round(tot_flops / (tot_us * 1e-6) / 1e12, 1)}
    return out


def one_dim_report(L, lf_synth, peaks, steps, flush):
    """layer480p with the one-dimensional selection (global block top-k over all
    KV blocks, no frame level; the ablation's variant) at the two-level call's
    kept-block budget: pooling, lf_select_blocks_1d and the attention."""
    import torch
    w = lf_synth.CONFIGS["layer480p"]
    shape = L.shape_from_workload(w)
    n_sel = L.lf_frames_selected(shape, w.chunk_index, w.topk_frames)
    kb2 = _kb(L, shape, w)
    keep = n_sel * kb2
    q, k, v = (t.cuda() for t in lf_synth.make_qkv(w))
    call = L.HSACall(shape, w.chunk_index, w.topk_frames, kb2)
    b = call.buf
    if b.list_cap < keep:
        raise RuntimeError("list capacity below the kept count")

    def select():
        L.lf_select_blocks_1d(shape, w.chunk_index, keep, b.q_pool, b.k_pool, b.block_list, b.block_count,
                              b.list_cap)
    for _ in range(3):
        call.pool(q, k)
        select()
        call.attend(q, k, v)
    torch.cuda.synchronize()
    flops = credited_flops(b.block_list.cpu().numpy(), b.block_count.cpu().numpy(), shape.frame_tokens,
                           shape.bpf, shape.head_dim, shape.n_cur)
    stream = torch.cuda.current_stream()
    E = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        e = E[i]
        e[0].record(stream)
        call.pool(q, k)
        e[1].record(stream)
        select()
        e[2].record(stream)
        call.attend(q, k, v)
        e[3].record(stream)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error: {st} {detail:#x}")

    def us(i0, i1):
        return statistics.mean(E[j][i0].elapsed_time(E[j][i1]) * 1e3 for j in range(steps))
    t, att = us(0, 3), us(2, 3)
    return {"us_per_call": round(t, 2),
            "kernels_us": {"pool": round(us(0, 1), 2), "select_1d": round(us(1, 2), 2), "attn": round(att, 2)},
            "kept_blocks_per_row": keep, "kept_tflop": round(flops / 1e12, 5),
            "tflops_call": round(flops / (t * 1e-6) / 1e12, 1),
            "attn_frac_of_bf16_peak": round(flops / (att * 1e-6) / 1e12 / peaks["bf16"], 4)}


def _time_us(fn, steps, flush, stream):
    import torch
    ts = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    return statistics.mean(ts)


def fp8_report(L, lf_synth, peaks, steps, flush):
    """layer480p through the FP8 attention (e4m3 q and k per token, bf16 softmax weights
    and v) on the bf16 call's lists. Its roofline peak mixes the two rates: QK^T runs on
    e4m3 tensor cores (the nominal 2x of bf16) and PV on bf16 ones, half the FLOPs each,
    so the time at peak is F/2/(2P) + F/2/P and the effective peak 4P/3 (P = the measured
    bf16 peak). k is quantised once per chunk (past frames do not change while a chunk
    denoises), q per call: both are reported."""
    import torch
    w = lf_synth.CONFIGS["layer480p"]
    shape = L.shape_from_workload(w)
    kb = _kb(L, shape, w)
    q, k, v = (t.cuda() for t in lf_synth.make_qkv(w))
    call = L.HSACall(shape, w.chunk_index, w.topk_frames, kb)
    call(q, k, v)
    b = call.buf
    q8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    k8 = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
    qs = torch.empty(q.shape[:-1], dtype=torch.float32, device="cuda")
    ks = torch.empty(k.shape[:-1], dtype=torch.float32, device="cuda")
    out8 = torch.empty_like(b.out)
    stream = torch.cuda.current_stream()
    quant_q = lambda: L.lf_quant_fp8_rows(q, q8, qs)
    quant_k = lambda: L.lf_quant_fp8_rows(k, k8, ks)
    attn8 = lambda: L.lf_block_sparse_attn_fp8(shape, q8, k8, qs, ks, v, b.block_list, b.block_count, b.list_cap,
                                               0.0, out8, call.workspace, call.tail_pieces)
    for _ in range(3):
        quant_q(); quant_k()
        # an NVTX range lets a profiler pick out the e4m3 attention launches
        torch.cuda.nvtx.range_push("lf_fp8_attn")
        attn8()
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error: {st} {detail:#x}")
    flops = credited_flops(b.block_list.cpu().numpy(), b.block_count.cpu().numpy(), shape.frame_tokens,
                           shape.bpf, shape.head_dim, shape.n_cur)
    t_q, t_k, t_a = (_time_us(f, steps, flush, stream) for f in (quant_q, quant_k, attn8))
    t_bf16 = _time_us(lambda: call.attend(q, k, v), steps, flush, stream)
    tf = flops / (t_a * 1e-6) / 1e12
    mixed_peak = peaks["bf16"] * 4.0 / 3.0
    return {"attn_fp8_us": round(t_a, 2), "attn_bf16_us_same_run": round(t_bf16, 2),
            "quant_q_us": round(t_q, 2), "quant_k_us_once_per_chunk": round(t_k, 2),
            "attn_fp8_tflops": round(tf, 1), "mixed_peak_tflops": round(mixed_peak, 1),
            "attn_fp8_frac_of_mixed_peak": round(tf / mixed_peak, 4),
            "quant_q_gbs": round((q.numel() * 3 + qs.numel() * 4) / (t_q * 1e-6) / 1e9, 1)}


def ivf_report(L, lf_synth, peaks, steps, flush, n_clusters=8, n_probe=2):
    """longvideo480p (60 memory frames) with the coarse frame index: index build (k-means
    over the frame means, once per appended chunk), probed frame selection against the
    exact one, and the recall of the exact top-k memory frames."""
    import torch
    w = lf_synth.CONFIGS["longvideo480p"]
    shape = L.shape_from_workload(w)
    kb = _kb(L, shape, w)
    q, k, v = (t.cuda() for t in lf_synth.make_qkv(w))
    call = L.HSACall(shape, w.chunk_index, w.topk_frames, kb)
    call.pool(q, k)
    b = call.buf
    idx = L.FrameIndex.empty(shape, n_clusters)
    sel_ivf = torch.empty_like(b.frame_sel)
    stream = torch.cuda.current_stream()
    build = lambda: L.lf_frame_index_build(shape, b.k_frame, idx, iters=25)
    probe = lambda: L.lf_select_frames_ivf(shape, w.chunk_index, w.topk_frames, idx, n_probe, b.q_pool,
                                           b.k_frame, sel_ivf)
    exact = lambda: L.lf_select_frames(shape, w.chunk_index, w.topk_frames, b.q_pool, b.k_frame, b.frame_sel)
    for _ in range(3):
        build(); probe(); exact()
    torch.cuda.synchronize()
    t_b, t_p, t_e = (_time_us(f, steps, flush, stream) for f in (build, probe, exact))
    n_sink, n_mem = shape.n_sink, shape.n_frames - shape.n_sink - shape.n_recent - shape.n_cur
    mem = lambda t: [set(f for f in r if n_sink <= f < n_sink + n_mem) for r in t.reshape(-1, t.shape[-1]).tolist()]
    a_, e_ = mem(sel_ivf.cpu()), mem(b.frame_sel.cpu())
    recall = sum(len(x & y) for x, y in zip(a_, e_)) / max(1, sum(len(y) for y in e_))
    return {"n_clusters": n_clusters, "n_probe": n_probe, "index_build_us": round(t_b, 2),
            "select_frames_ivf_us": round(t_p, 2), "select_frames_exact_us": round(t_e, 2),
            "recall_of_exact_memory_frames": round(recall, 4)}


def run_ours(a):
    import numpy as np
    import torch

    dist, rank, ws, local = _dist()
    torch.cuda.set_device(local)
    import block_sparse_attention_lf_b200 as L
    import lf_synth

    w, shape, q_h, k_h, v_h, units = _rank_inputs(L, lf_synth, a.workload, rank, ws, a.strong)
    if shape is None:  # more ranks than units: this rank idles but takes every collective step
        _idle_rank(a, dist, ws)
        return
    kb = _kb(L, shape, w)
    q, k, v = q_h.cuda(), k_h.cuda(), v_h.cuda()
    call = L.HSACall(shape, w.chunk_index, w.topk_frames, kb)
    b = call.buf
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    for _ in range(max(3, a.warmup)):
        call(q, k, v)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    if st != 0:
        raise SystemExit(f"device error after warm-up: {st} {detail:#x}")
    flops = credited_flops(b.block_list.cpu().numpy(), b.block_count.cpu().numpy(),
                           shape.frame_tokens, shape.bpf, shape.head_dim, shape.n_cur)

    # The timed call: events only around it (the selection and the attention are launched as
    # programmatic dependents of the kernel before them, which events in between would stop).
    EC = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for i in range(a.steps):
            flush.zero_()
            EC[i][0].record(stream)
            call(q, k, v)
            EC[i][1].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    if dist is not None:
        dist.barrier()
    st, detail = L.lf_get_device_error()
    if st != 0:
        raise SystemExit(f"device error in the timed region: {st} {detail:#x}")
    step_ms = [e0.elapsed_time(e1) for e0, e1 in EC]
    # per-kernel times: a second pass with events between the kernels
    E = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(a.steps)]
    for i in range(a.steps):
        flush.zero_()
        e = E[i]
        e[0].record(stream)
        call.pool(q, k)
        e[1].record(stream)
        call.select()
        e[2].record(stream)
        e[3].record(stream)
        call.attend(q, k, v)
        e[4].record(stream)
    torch.cuda.synchronize()

    def mean_ms(i0, i1):
        return statistics.mean(E[s][i0].elapsed_time(E[s][i1]) for s in range(a.steps))

    t_pool, t_sel, t_attn = mean_ms(0, 1), mean_ms(1, 2), mean_ms(3, 4)
    # attention alone, back to back with a warm L2 (K/V of the call stay resident)
    ew = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    for s0, s1 in ew:
        s0.record(stream)
        call.attend(q, k, v)
        s1.record(stream)
    torch.cuda.synchronize()
    t_attn_warm = statistics.mean(s0.elapsed_time(s1) for s0, s1 in ew)
    t_step = statistics.mean(step_ms)
    t_step_max = _max_over_ranks(dist, t_step)
    total_flops = _reduce_over_ranks(dist, flops, "sum")  # every rank's units
    value = total_flops / (t_step_max * 1e-3) / 1e12

    # ---- end to end through the public API with pinned host buffers
    qp_, kp_, vp_ = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    out_h = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()
    e2e_steps = max(3, min(a.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        flush.zero_()
        ev[i][0].record(stream)
        q.copy_(qp_, non_blocking=True)
        k.copy_(kp_, non_blocking=True)
        v.copy_(vp_, non_blocking=True)
        call(q, k, v)
        out_h.copy_(b.out, non_blocking=True)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    t_e2e_serial = statistics.mean(s.elapsed_time(t) for s, t in ev)
    # The same call pipelined by head groups through the same public API (HSACall on each
    # group's units, unit_view slices): group g's inputs cross PCIe while group g-1 computes
    # and group g-2's output returns, so the copies hide the compute.
    n_groups = min(E2E_GROUPS, shape.batch * shape.heads)
    groups = []
    for g in range(n_groups):
        sub, u0, u1 = L.shard_shape(shape, n_groups, g)
        if sub is None:
            continue
        groups.append((L.HSACall(sub, w.chunk_index, w.topk_frames, kb),
                       [L.unit_view(t, u0, u1) for t in (q, k, v)],
                       [L.unit_view(t, u0, u1) for t in (qp_, kp_, vp_)],
                       L.unit_view(out_h, u0, u1)))
    s_h2d, s_cmp, s_d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for gc, dev, _, _ in groups:  # warm the group calls
        gc(*dev)
    torch.cuda.synchronize()
    evp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        flush.zero_()
        evp[i][0].record(stream)
        for st_ in (s_h2d, s_cmp, s_d2h):
            st_.wait_event(evp[i][0])
        for gc, dev, host, oh in groups:
            with torch.cuda.stream(s_h2d):
                for d_, h_ in zip(dev, host):
                    d_.copy_(h_, non_blocking=True)
                copied = torch.cuda.Event()
                copied.record(s_h2d)
            s_cmp.wait_event(copied)
            gc(*dev, stream=s_cmp)
            done = torch.cuda.Event()
            done.record(s_cmp)
            s_d2h.wait_event(done)
            with torch.cuda.stream(s_d2h):
                oh.copy_(gc.buf.out, non_blocking=True)
        for st_ in (s_h2d, s_cmp, s_d2h):
            stream.wait_stream(st_)
        evp[i][1].record(stream)
    torch.cuda.synchronize()
    st, detail = L.lf_get_device_error()
    if st != 0:
        raise SystemExit(f"device error in the end-to-end run: {st} {detail:#x}")
    t_e2e = _max_over_ranks(dist, statistics.mean(s.elapsed_time(t) for s, t in evp))
    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = b.out.numel() * 2

    peaks = _peaks()
    attn_tflops = flops / (t_attn * 1e-3) / 1e12
    pool_bytes = (q.numel() + k.numel()) * 2 + (b.q_pool.numel() + b.k_pool.numel() + b.k_frame.numel()) * 4
    sel_bytes = ((b.q_pool.numel() + b.k_frame.numel() + b.k_pool.numel()) * 4
                 + (b.frame_sel.numel() + b.block_count.numel()) * 4
                 + shape.batch * shape.heads * shape.Rq * b.list_cap * 4)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": t_step_max, "higher_is_better": True,
        "scaling": "strong" if (a.strong and ws > 1) else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (lf_synth, seeded; stands in for the pages' VBench 480p rollouts)",
        "config": dict(_config(w, kb), global_batch=w.batch * (1 if (a.strong or ws == 1) else ws),
                       parallelism=(f"(batch, head) units split over {ws} GPU(s), no exchange; "
                                    f"rank 0 units [{units[0]}, {units[1]})")),
        "us_per_call": t_step_max * 1e3,
        "us_p10_p90": [_pct(step_ms, 10) * 1e3, _pct(step_ms, 90) * 1e3],
        "attn_us_warm_l2": t_attn_warm * 1e3,
        "kernels_us": {"pool": t_pool * 1e3, "select": t_sel * 1e3, "block_sparse_attn": t_attn * 1e3},
        "kept_tflop_per_call": flops / 1e12,
        "attn_tflops": attn_tflops,
        "attn_frac_of_bf16_peak": attn_tflops / peaks["bf16"],
        "pool_gbs": pool_bytes / (t_pool * 1e-3) / 1e9,
        "pool_frac_of_hbm": pool_bytes / (t_pool * 1e-3) / 1e9 / peaks["hbm"],
        "select_gbs": sel_bytes / (t_sel * 1e-3) / 1e9,
        "select_over_attn": (t_pool + t_sel) / t_attn,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16"],
                     "traffic": _attn_traffic(),
                     "peak_source": f"{peaks['source']} bf16 dense burst (MEASURED_PEAKS.json)"},
        "e2e": {"value": total_flops / (t_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": t_e2e,
                "pipeline": f"{len(groups)} head groups, copies and compute on separate streams",
                "ms_per_step_unpipelined": t_e2e_serial},
        "gpu_launches": call.launches_per_call * a.steps,
        "clocks": clk.summary(),
        "wall_s_timed_region": wall,
    }
    extra = (("layer480p_1d", one_dim_report), ("layer480p_fp8", fp8_report), ("longvideo480p_ivf", ivf_report))
    if rank == 0 and a.only_report == "cached_pooled_keys":
        mc = measure_call(L, shape, w.chunk_index, w.topk_frames, kb, q, k, v, a.config_steps, 3, flush, cached=True)
        line["cached_pooled_keys"] = _summary(mc, peaks)
    elif rank == 0 and a.only_report:
        line["configs"] = {}
        for key, fn in extra:
            if key == a.only_report:
                line["configs"][key] = fn(L, lf_synth, peaks, a.config_steps, flush)
    elif rank == 0 and not a.no_configs:
        mc = measure_call(L, shape, w.chunk_index, w.topk_frames, kb, q, k, v, a.config_steps, 3, flush, cached=True)
        line["cached_pooled_keys"] = dict(_summary(mc, peaks), note=(
            "pooled keys of past frames kept from a first full pooling; each call re-pools the "
            "current chunk's frames and the queries (lf_pool_range)"))
        line["configs"] = config_report(L, lf_synth, peaks, a.config_steps, flush)
        for key, fn in extra:
            try:
                line["configs"][key] = fn(L, lf_synth, peaks, a.config_steps, flush)
            except Exception as e:  # an extra report never costs the main line
                line["configs"][key] = {"error": repr(e)[:200]}
    if rank == 0 and ws == 1 and not a.no_cpu_baseline:
        r = _oracle_sample(w, a.cpu_budget_s, q_h, k_h, v_h)
        line["cpu_baseline"] = {"value": r["flops"] / r["t_call"] / 1e12, "unit": "TFLOP/s",
                                "cores": 1, "kind": "oracle", "sample": r["sample"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    a = _args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
