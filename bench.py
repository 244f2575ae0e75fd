#!/usr/bin/env python
"""Benchmark of the QSA hot path on B200.

Default (N=1): the largest single-GPU workload, a batched variable-length bf16
prefill: batch 8, padded length 16384, left pads uniform in [0, 2048], 32 query /
4 KV heads, head_dim 128, 8 indexer heads of dim 64, block 128, top-k 16 (+ the
trailing block). A step is one pass of the whole path (compress -> score/top-k ->
sparse attention) over that batch, inputs resident in HBM, L2 flushed between
steps. Also measured:
  workloads -- the same step on the long 64K prefill (planted blocks, top-k 64) and
               on the 8K prefill (16 / 2 heads, block 64, top-k 32), each with its
               attention kernel's roofline;
  projection -- the projections + RoPE (qsa_project) over the headline batch's rows at
               hidden size 2048, with cuBLAS's time for the bare GEMM as context;
  e2e       -- the headline step through qsa_forward with pinned HOST buffers, the
               host->device copy of the inputs (one copy from a pinned arena) and
               the device->host read of the output inside the timed region;
  decode    -- one decode step for 64 sequences with caches of 4096..32768 tokens
               (CUDA-graph replay, L2 flushed between steps), plus its attention
               kernel against the HBM roofline; the same at head_dim 256, and the
               step with the K/V cache offloaded to host memory;
  roofline  -- the attention kernel's selected-token FLOPs over its CUDA-event time
               against the measured bf16 tensor-core peak;
  cpu_baseline -- the fp64 CPU oracle on a bounded random sample of query rows.
With --gpus N under torchrun each rank runs its own replica of the workload (the
path has no cross-sequence exchange); value = all ranks' tokens / max-over-ranks time.
--impl reference times the oracle itself as the reference arm.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QSA prefill tokens/s & decode µs/step at 1 B200; % of TC / HBM roofline"


class L2Flush:
    """Evict L2 between timed steps: write a buffer larger than L2, then read another
    one, so that the written lines are back in HBM before the timed region starts
    (otherwise their write-back would compete with an HBM-bound kernel)."""

    def __init__(self, device, nbytes):
        import torch
        self.w = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
        self.r = torch.zeros(nbytes // 4, dtype=torch.float32, device=device)
        self.sink = torch.zeros((), dtype=torch.float32, device=device)

    def zero_(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="bf16_prefill_varlen_b8_s16384_leftpad")
    p.add_argument("--extra-workloads", default="bf16_prefill_s65536_planted,bf16_prefill_s8192,bf16_prefill_s8192_hd256",
                   help="comma-separated prefill workloads measured beside the headline ('' for none)")
    p.add_argument("--decode-workload", default="bf16_decode_b64_l4k_32k")
    p.add_argument("--more-decode-workloads", default="bf16_decode_b64_l4k_32k_hd256",
                   help="comma-separated decode workloads measured beside the main one ('' for none)")
    p.add_argument("--no-offload", action="store_true", help="skip the offloaded decode step")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-projection", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--batch", type=int, default=0,
                   help="override the headline workload's batch (a smaller case of the same shape, for "
                        "profiling captures); 0 keeps the workload's own")
    return p.parse_args(argv)


# --------------------------------------------------------------------------- counting
def attended_pairs(w, inp):
    """Exact (query, key) pairs per head summed over real query rows: each row t sees
    min(n_c, k) whole blocks plus its trailing range of (t + 1 - n_c * B) tokens."""
    import numpy as np
    total = 0
    score_pairs = 0
    for b in range(w.batch):
        L = int(inp["kv_len"][b])
        q_first = int(inp["q_first"][b])
        n_q = inp["q"].shape[1]
        t = np.arange(max(0, q_first), min(L, q_first + n_q), dtype=np.int64)
        n_c = (t + 1) // w.block
        total += int((np.minimum(n_c, w.topk) * w.block + (t + 1 - n_c * w.block)).sum())
        score_pairs += int(n_c.sum())
    return total, score_pairs


def tc_executed_flops(w, inp, sel):
    """Tensor-core FLOPs the prefill attention kernel (k_attn_tc) executes, masked work
    included: a unit's two 128-row tiles each hold T = 128 / G consecutive query rows
    of one KV head, and a tile multiplies (QK^T and PV, 128 rows x 128 keys x d each)
    every 128-key chunk of the key range in which any of its rows sees a key -- of a
    selected block or of its trailing range. sel: the selection the kernel read,
    [batch][n_q][k]."""
    import numpy as np
    G = w.Hq // w.Hkv
    T = 128 // G
    chunk = 128
    per = 4.0 * 128 * chunk * w.d  # one tile x one chunk: QK^T and PV
    total = 0
    n_q = inp["q"].shape[1]
    for b in range(w.batch):
        L, qf = int(inp["kv_len"][b]), int(inp["q_first"][b])
        s = np.asarray(sel[b])
        n_tiles = (n_q + T - 1) // T
        n_ch = (max(L, 1) + chunk - 1) // chunk
        need = np.zeros((n_tiles, n_ch + 1), dtype=bool)
        r = np.arange(n_q)
        t = qf + r
        ok = (t >= 0) & (t < L)
        r, t = r[ok], t[ok]
        tile = r // T
        n_c = (t + 1) // w.block
        blk = s[r]
        rows_i, cols_i = np.nonzero((blk >= 0) & (blk < n_c[:, None]))
        first, last = blk[rows_i, cols_i] * w.block, blk[rows_i, cols_i] * w.block + w.block - 1
        for off in range(0, w.block + chunk, chunk):  # every chunk a selected block touches
            c = np.minimum((first + off) // chunk, last // chunk)
            need[tile[rows_i], c] = True
        lo = n_c * w.block
        has_tr = lo <= t
        for off in range(0, w.block + chunk, chunk):  # every chunk the trailing range touches
            c = np.minimum((lo + off) // chunk, t // chunk)
            need[tile[has_tr], c[has_tr]] = True
        total += int(need.sum())
    return total * per * w.Hkv


def real_rows(inp):
    n = 0
    for b in range(inp["q"].shape[0]):
        L, qf, n_q = int(inp["kv_len"][b]), int(inp["q_first"][b]), inp["q"].shape[1]
        n += max(0, min(L, qf + n_q) - max(0, qf))
    return n


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def file_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel_key):
    """dram bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
        ent = tab[kernel_key]
        if ent.get("source_sha") != file_sha(ent["source"]):
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"qsa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()
        return False

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- CPU oracle
def cpu_oracle_rate(w, inp, seconds, seed=0):
    """fp64 oracle over a seeded uniform sample of real query rows; rows/s == tokens/s."""
    import numpy as np

    import oracle
    g = np.random.default_rng(seed)
    rows_all = []
    for b in range(w.batch):
        L, qf, n_q = int(inp["kv_len"][b]), int(inp["q_first"][b]), inp["q"].shape[1]
        rows_all += [(b, r) for r in range(max(0, -qf), min(n_q, L - qf))]

    def run(n):
        idx = g.choice(len(rows_all), size=min(n, len(rows_all)), replace=False)
        by_b = {}
        for i in idx:
            b, r = rows_all[i]
            by_b.setdefault(b, []).append(r)
        t0 = time.perf_counter()
        oracle.run(w, inp, rows={b: sorted(v) for b, v in by_b.items()})
        return len(idx), time.perf_counter() - t0

    # A call has a fixed part (the workload's block means, set-up) besides its per-row
    # work: two pilot sizes separate them, so the main sample lasts about `seconds`.
    n1, d1 = run(32)
    n2, d2 = run(min(256, len(rows_all)))
    per_row = max((d2 - d1) / max(n2 - n1, 1), d2 / max(n2, 1) / 16, 1e-6)
    fixed = max(d1 - per_row * n1, 0.0)
    n_main = int(min(len(rows_all), max(n2, (seconds - fixed) / per_row)))
    n, dt = run(n_main)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n} query rows drawn uniformly (seed {seed}) from the {len(rows_all)} real rows of "
                      f"{w.name}; fp64 C oracle, OpenMP over rows; {dt:.1f} s"}


# --------------------------------------------------------------------------- GPU arms
def bench_prefill(args, w, inp, dist_info, with_e2e=True):
    import torch

    from block_sparse_long_15_b200 import qsa
    from block_sparse_long_15_b200.runner import QSAPrefill, to_device
    dev = torch.cuda.current_device()
    p = QSAPrefill(w, inp)
    cfg, t, ws = p.cfg, p.t, p.ws
    kv_cap = t["k_cache"].shape[2]
    stream = torch.cuda.current_stream()
    flush = L2Flush(dev, L2_FLUSH_BYTES)

    def step(evs=None):
        """One prefill through the public call: qsa_forward chains compress -> score ->
        attention as programmatic dependents (one entry, four launches)."""
        if evs:
            evs[0].record()
        qsa.qsa_forward(cfg, qsa.QSA_PREFILL, t, ws)
        if evs:
            evs[1].record()

    def stages(evs=None):
        """The same work as three stage calls, each timed on its own."""
        if evs:
            evs[0].record()
        qsa.qsa_compress_blocks(cfg, t["ki_cache"], t["kv_start"], t["kv_len"], t["kbar_cache"])
        if evs:
            evs[1].record()
        qsa.qsa_index_score_topk(cfg, t["qi"], t["kbar_cache"], t["kv_len"], t["q_first"], kv_cap,
                                 t["sel"], ws)
        if evs:
            evs[2].record()
        qsa.qsa_sparse_attn(cfg, t["q"], t["k_cache"], t["v_cache"], t["sel"], t["kv_start"], t["kv_len"],
                            t["q_first"], t["out"], ws)
        if evs:
            evs[3].record()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(dev) as clk:
        # the same load before and after the timed steps, so that the 200 ms clock
        # samples bracket the (much shorter) timed region
        load_for(0.5, lambda: (flush.zero_(), step()))
        barrier(dist_info)
        torch.cuda.synchronize()
        n0 = qsa.qsa_kernel_launch_count()
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
        launches = qsa.qsa_kernel_launch_count() - n0
        barrier(dist_info)
        torch.cuda.synchronize()
        # stage times: the same steps as three separately timed stage calls
        for i in range(args.steps):
            flush.zero_()
            stages(sev[i])
        torch.cuda.synchronize()
        load_for(0.3, lambda: (flush.zero_(), step()))
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    stage_ms = [[e[j].elapsed_time(e[j + 1]) for e in sev] for j in range(3)]
    assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK

    e2e = None
    if with_e2e and not args.no_e2e:
        e2e = bench_prefill_e2e(args, w, inp, p, stream)
    return dict(step_ms=step_ms, stage_ms=stage_ms, launches=launches, clocks=clk.summary(), e2e=e2e,
                kernel=qsa.qsa_attn_kernel_name(cfg), sel=t["sel"].cpu())


def load_for(seconds, fn):
    """Keep the GPU busy with fn() for about `seconds` (untimed)."""
    import torch
    t_end = time.perf_counter() + seconds
    while time.perf_counter() < t_end:
        for _ in range(8):
            fn()
        torch.cuda.synchronize()


class PinnedArena:
    """Inputs of one step packed into one pinned host buffer and one device buffer of
    the same layout (each tensor 256-byte aligned), so that a step's upload is a
    single host->device copy."""

    def __init__(self, tensors, device):
        import torch
        self.layout, off = {}, 0
        for name, t in tensors.items():
            n = t.numel() * t.element_size()
            self.layout[name] = (off, n, t.dtype, tuple(t.shape))
            off += (n + 255) // 256 * 256
        self.host = torch.empty(off, dtype=torch.uint8).pin_memory()
        for name, t in tensors.items():
            self.view(self.host, name).copy_(t)
        self.device = device
        self.nbytes = off

    def view(self, buf, name):
        off, n, dt, shape = self.layout[name]
        return buf[off:off + n].view(dt).view(shape)

    def device_buffer(self):
        import torch
        return torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)


E2E_SETS = 3  # device buffer sets of the end-to-end serving loop


def bench_prefill_e2e(args, w, inp, p, stream):
    """The step through qsa_forward (the public call) from pinned host inputs to a pinned
    host output, every copy inside the timed region. Steps run as a serving loop would:
    E2E_SETS sets of device buffers, uploads on one stream, qsa_forward on another,
    downloads on a third, so that step i + 1's upload overlaps step i's compute and
    download (the host link is full duplex and the copy engines run beside the SMs).
    With two sets, step i + 2's upload would wait for step i's download, putting
    upload + compute + download on the critical path of every two steps; with three,
    the upload alone bounds the step. Every step still uploads all of its inputs -- one
    copy of the packed arena -- and reads its result back. Reported: throughput (ms per
    step over the pipelined run) and the latency of one step run alone."""
    import torch

    from block_sparse_long_15_b200 import qsa
    from block_sparse_long_15_b200.runner import QSAPrefill
    names = {"q": "q", "qi": "qi", "k": "k_cache", "v": "v_cache", "ki": "ki_cache",
             "kv_start": "kv_start", "kv_len": "kv_len", "q_first": "q_first"}
    arena = PinnedArena({k: inp[k].contiguous() for k in names}, torch.cuda.current_device())
    sets, bufs = [p] + [QSAPrefill(w, inp) for _ in range(E2E_SETS - 1)], []
    for x in sets:  # the buffer set's inputs become views of its device arena
        buf = arena.device_buffer()
        for name, dst in names.items():
            x.t[dst] = arena.view(buf, name)
        bufs.append(buf)
    outs = [torch.empty(p.t["out"].shape, dtype=p.t["out"].dtype).pin_memory() for _ in sets]
    h2d = arena.nbytes
    d2h = outs[0].numel() * outs[0].element_size()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    free = [None] * E2E_SETS  # per buffer set: event after its last download

    def step(i):
        k = i % E2E_SETS
        x, o = sets[k], outs[k]
        if free[k] is not None:
            s_in.wait_event(free[k])
        with torch.cuda.stream(s_in):
            bufs[k].copy_(arena.host, non_blocking=True)
        up = torch.cuda.Event()
        up.record(s_in)
        s_run.wait_event(up)
        qsa.qsa_forward(x.cfg, qsa.QSA_PREFILL, x.t, x.ws, s_run)
        done = torch.cuda.Event()
        done.record(s_run)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            o.copy_(x.t["out"], non_blocking=True)
            free[k] = torch.cuda.Event()
            free[k].record(s_out)

    for i in range(max(E2E_SETS, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    # latency of one step alone
    lat = []
    for i in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        step(i)
        b.record(s_out)
        torch.cuda.synchronize()
        lat.append(a.elapsed_time(b))
    # throughput of the pipelined loop
    n = max(5, args.steps // 2)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(n):
        step(i)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    for x in sets:
        assert qsa.qsa_read_device_status(x.ws) == qsa.QSA_OK
    for o in outs[1:]:
        assert torch.equal(outs[0].view(torch.int16), o.view(torch.int16))
    return dict(ms=a.elapsed_time(b) / n, h2d=h2d, d2h=d2h, latency_ms=statistics.median(lat),
                copies_per_step={"h2d": 1, "d2h": 1})


PROJ_HIDDEN = 2048  # Qwen4ExpTextConfig's hidden_size default


def bench_projection(args, w, peaks, peak_src):
    """The projection stage (qsa_project: q/k/v/indexer projections + RoPE, one tcgen05
    GEMM) over every row of the workload's padded batch at hidden size 2048, weights and
    hidden states synthetic (N(0,1) rows, N(0,1)/sqrt(hidden) weights, bf16), L2 flushed
    between launches. cuBLAS's time for the same GEMM without the RoPE epilogue is
    reported beside it as context."""
    import torch

    from block_sparse_long_15_b200 import qsa
    dev = torch.cuda.current_device()
    rows, hidden = w.batch * w.seq, PROJ_HIDDEN
    n_out = w.Hq * w.d + 2 * w.Hkv * w.d + w.Hi * w.di + w.di
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn(w.batch, w.seq, hidden, device="cuda", generator=g).to(torch.bfloat16)
    wt = (torch.randn(n_out, hidden, device="cuda", generator=g) / hidden ** 0.5).to(torch.bfloat16)
    bf = torch.bfloat16
    q = torch.empty(w.batch, w.seq, w.Hq, w.d, dtype=bf, device="cuda")
    qi = torch.empty(w.batch, w.seq, w.Hi, w.di, dtype=bf, device="cuda")
    k = torch.empty(w.batch, w.Hkv, w.seq, w.d, dtype=bf, device="cuda")
    v = torch.empty_like(k)
    ki = torch.empty(w.batch, w.seq, w.di, dtype=bf, device="cuda")
    q_first = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    cfg = qsa.config_for(w)
    pc = qsa.qsa_proj_config_t(hidden, 1e6, w.d, w.di)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    flush = L2Flush(dev, L2_FLUSH_BYTES)

    def timed(fn, n):
        out = []
        for _ in range(n):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            out.append(a.elapsed_time(b))
        return statistics.median(out)

    run = lambda: qsa.qsa_project(cfg, pc, x, wt, q_first, q, qi, k, v, ki, 0, ws)
    for _ in range(args.warmup):
        run()
    ms = timed(run, max(5, args.steps))
    assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK
    y = torch.empty(rows, n_out, dtype=bf, device="cuda")
    gemm = lambda: torch.matmul(x.view(rows, hidden), wt.t(), out=y)
    for _ in range(args.warmup):
        gemm()
    ms_lib = timed(gemm, max(5, args.steps))
    flops = 2.0 * rows * hidden * n_out
    sustained = ms >= LONG_STEP_MS
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    ach = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "rows": rows, "hidden_size": hidden, "n_out": n_out, "ms": ms,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                         "peak_source": (f"bf16_tflops_sustained of {peak_src}" if sustained
                                         else f"bf16_tflops (burst) of {peak_src}"),
                         "flops_per_launch": flops},
            "cublas_gemm_ms": ms_lib, "cublas_gemm_tflops": flops / (ms_lib * 1e-3) / 1e12}


def decode_kernel_bytes(w, inp):
    """Algorithmic bytes of the decode attention kernel: K and V of every attended token
    of each KV head, the query and the output rows (bf16)."""
    esz = 2 if w.dtype == "bf16" else 4
    total = 0
    for b in range(w.batch):
        L = int(inp["kv_len"][b])
        n_c = L // w.block
        toks = min(n_c, w.topk) * w.block + (L - n_c * w.block)
        total += toks * w.Hkv * w.d * esz * 2 + 2 * w.Hq * w.d * esz
    return total


def decode_step_bytes(w, inp):
    """Whole decode step: attention bytes + k̄ rows scored + indexer query + appended token."""
    esz = 2 if w.dtype == "bf16" else 4
    total = decode_kernel_bytes(w, inp)
    for b in range(w.batch):
        L = int(inp["kv_len"][b])
        total += (L // w.block) * w.di * 4 + w.Hi * w.di * esz + (2 * w.Hkv * w.d + w.di) * esz * 2
    return total


def bench_decode_offload(args, wd, inp, peaks):
    """The decode step with the attention K/V cache in page-locked host memory
    (qsa_decode_offload): selection on the device, then only the attended blocks cross
    the host link into a device staging cache. Median of a few steps, L2 flushed."""
    import torch

    from block_sparse_long_15_b200 import qsa
    from block_sparse_long_15_b200.runner import QSADecodeOffload
    d = QSADecodeOffload(wd, inp)
    flush = L2Flush(torch.cuda.current_device(), L2_FLUSH_BYTES)
    for _ in range(max(2, args.warmup)):
        d()
    torch.cuda.synchronize()
    ts = []
    for _ in range(max(5, args.steps)):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        d()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    assert d.status() == qsa.QSA_OK
    kb = decode_kernel_bytes(wd, inp)
    ms = statistics.median(ts)
    return {"workload": wd.name, "ms_per_step": ms, "host_link_bytes_per_step": kb,
            "host_link_gbs": kb / (ms * 1e-3) / 1e9,
            "note": "K/V cache in page-locked host memory; the attended blocks cross the host link each step"}


def bench_decode(args, wd, dist_info, peaks, inp=None):
    import torch

    from block_sparse_long_15_b200 import qsa, workloads as W
    from block_sparse_long_15_b200.runner import QSADecode
    if inp is None:
        inp = W.make_inputs(wd)
    d = QSADecode(wd, inp)
    dev = torch.cuda.current_device()
    flush = L2Flush(dev, L2_FLUSH_BYTES)
    for _ in range(3):
        d()
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_OK
    # whole step as a CUDA graph
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        d()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            d()
    torch.cuda.synchronize()
    n = max(20, args.steps * 5)
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for _ in range(args.warmup):
        flush.zero_()
        g.replay()
    for i in range(n):
        flush.zero_()
        e0[i].record()
        g.replay()
        e1[i].record()
    torch.cuda.synchronize()
    step_us = statistics.median(a.elapsed_time(b) for a, b in zip(e0, e1)) * 1e3
    # the attention kernel alone (stage call, captured as its own graph so that host
    # work such as tensor-map encoding stays outside the GPU time), same inputs
    cfg = d.cfg
    q_first = (d.t["kv_len"] - 1).contiguous()
    ga = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(ga, stream=side):
            qsa.qsa_sparse_attn(cfg, d.t["q"], d.t["k_cache"], d.t["v_cache"], d.t["sel"], d.t["kv_start"],
                                d.t["kv_len"], q_first, d.t["out"], d.ws)
    torch.cuda.synchronize()
    a0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    a1 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for i in range(n + args.warmup):
        flush.zero_()
        if i >= args.warmup:
            a0[i - args.warmup].record()
        ga.replay()
        if i >= args.warmup:
            a1[i - args.warmup].record()
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_OK
    attn_us = statistics.median(a.elapsed_time(b) for a, b in zip(a0, a1)) * 1e3
    del ga
    kb = decode_kernel_bytes(wd, inp)
    sb = decode_step_bytes(wd, inp)
    del g
    return {"workload": wd.name, "us_per_step": step_us, "graph": True,
            "step_bytes": sb, "step_gbs": sb / (step_us * 1e-6) / 1e9,
            "kernel": qsa.qsa_attn_kernel_name(cfg, qsa.QSA_DECODE),
            "roofline": {"bound": "hbm", "achieved": kb / (attn_us * 1e-6) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": kb / (attn_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                         "traffic": ncu_traffic("attn_decode:" + wd.name), "kernel_us": attn_us,
                         "bytes_per_launch": kb},
            "l2": "flushed between steps (256 MiB write, then 256 MiB read)"}


# --------------------------------------------------------------------------- distributed
def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return None
    import torch
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    import datetime
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return {"rank": rank, "world": ws, "backend": backend}


def barrier(info):
    if info is None:
        return
    import torch.distributed as dist
    dist.barrier()


def max_over_ranks(x: float, info) -> float:
    if info is None:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if info["backend"] == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(ms_per_step_rank: float, tokens_per_rank: int, info):
    """Whole-job throughput: all ranks' tokens over the slowest rank's step time."""
    world = 1 if info is None else info["world"]
    ms = max_over_ranks(ms_per_step_rank, info)
    return ms, world * tokens_per_rank / (ms * 1e-3)


# --------------------------------------------------------------------------- main
def main(argv=None):
    args = parse_args(argv)
    info = dist_setup(args)
    rank = 0 if info is None else info["rank"]
    n_gpus = 1 if info is None else info["world"]
    from block_sparse_long_15_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if args.batch > 0 and args.batch != w.batch:
        w = w.replace(batch=args.batch, name=f"{w.name}__b{args.batch}")
    if args.impl == "reference":
        return main_reference(args, w, info, rank, n_gpus)

    import torch
    from block_sparse_long_15_b200 import build
    build.build()
    peaks, peak_src = load_peaks()
    inp = W.make_inputs(w)
    r = bench_prefill(args, w, inp, info)
    head = prefill_record(w, inp, r, peaks, peak_src, info)
    out = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": n_gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seq, "num_attention_heads": w.Hq,
                   "num_key_value_heads": w.Hkv, "head_dim": w.d, "indexer_n_heads": w.Hi,
                   "indexer_head_dim": w.di, "indexer_compress_ratio": w.block,
                   "indexer_budget": w.topk * w.block, "left_pad_max": w.pad_max, "seed": w.seed,
                   "real_tokens": real_rows(inp),
                   "l2": "flushed between steps (256 MiB write, then 256 MiB read)",
                   "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU"},
        "roofline": head["roofline"],
        "gpu_launches": r["launches"], "clocks": r["clocks"],
    }
    if r["e2e"]:
        e = r["e2e"]
        e_ms, e_val = aggregate(e["ms"], real_rows(inp), info)
        out["e2e"] = {"value": e_val, "unit": "tokens/s", "h2d_bytes_per_step": e["h2d"],
                      "d2h_bytes_per_step": e["d2h"], "ms_per_step": e_ms, "pipelined": True,
                      "latency_ms": e["latency_ms"], "copies_per_step": e["copies_per_step"]}
    cpu_inp = inp if (rank == 0 and n_gpus == 1 and not args.no_cpu_baseline) else None
    del r["sel"]
    torch.cuda.empty_cache()
    extra = {}
    for name in [x for x in args.extra_workloads.split(",") if x]:
        wx = W.WORKLOADS[name]
        ix = W.make_inputs(wx)
        rx = bench_prefill(args, wx, ix, info, with_e2e=False)
        rec = prefill_record(wx, ix, rx, peaks, peak_src, info)
        rec["clocks"] = rx["clocks"]
        rec["gpu_launches"] = rx["launches"]
        extra[name] = rec
        del rx, ix
        torch.cuda.empty_cache()
    if extra:
        out["workloads"] = extra
    if not args.no_projection:
        out["projection"] = bench_projection(args, w, peaks, peak_src)
        torch.cuda.empty_cache()
    if not args.no_decode:
        wd = W.WORKLOADS[args.decode_workload]
        dinp = W.make_inputs(wd)
        dec = bench_decode(args, wd, info, peaks, dinp)
        dec["us_per_step"] = max_over_ranks(dec["us_per_step"], info)
        out["decode"] = dec
        more = {}
        for name in [x for x in args.more_decode_workloads.split(",") if x]:
            dm = bench_decode(args, W.WORKLOADS[name], info, peaks)
            dm["us_per_step"] = max_over_ranks(dm["us_per_step"], info)
            more[name] = dm
            torch.cuda.empty_cache()
        if more:
            out["decode_more"] = more
        if not args.no_offload and info is None:  # single-GPU runs: it pins a 2 GB host cache
            out["decode_offload"] = bench_decode_offload(args, wd, dinp, peaks)
            torch.cuda.empty_cache()
    if cpu_inp is not None:
        out["cpu_baseline"] = cpu_oracle_rate(w, cpu_inp, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if info is not None:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# A prefill step that runs this long back to back is timed as "inside a long step":
# its kernels run at the power-capped sustained clock, so its roofline takes the
# sustained tensor peak; shorter steps take the burst peak. Both fractions are
# reported.
LONG_STEP_MS = 2.0


def prefill_record(w, inp, r, peaks, peak_src, info):
    """Throughput of a prefill step and its attention kernel's roofline (selected-token
    FLOPs only; masked tensor-core work is never counted)."""
    ms_rank = statistics.mean(r["step_ms"])
    ms, value = aggregate(ms_rank, real_rows(inp), info)
    pairs, score_pairs = attended_pairs(w, inp)
    attn_flops = 4.0 * w.d * w.Hq * pairs
    score_flops = 2.0 * w.Hi * w.di * score_pairs
    attn_ms = statistics.mean(r["stage_ms"][2])
    achieved = attn_flops / (attn_ms * 1e-3) / 1e12
    sustained = ms >= LONG_STEP_MS
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    executed = tc_executed_flops(w, inp, r["sel"]) if r["kernel"] == "tcgen05" else None
    return {
        "workload": w.name, "value": value, "unit": "tokens/s", "ms_per_step": ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "frac_of_burst": achieved / peaks["bf16_tflops"],
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "traffic": ncu_traffic("attn_prefill:" + w.name),
                     "peak_source": (f"bf16_tflops_sustained of {peak_src} (step of {ms:.1f} ms run back to back)"
                                     if sustained else f"bf16_tflops (burst) of {peak_src}"),
                     "kernel": r["kernel"], "kernel_ms": attn_ms, "flops_per_launch": attn_flops,
                     "stage_ms": {"compress": statistics.mean(r["stage_ms"][0]),
                                  "score_topk": statistics.mean(r["stage_ms"][1]),
                                  "sparse_attn": attn_ms},
                     "score_flops_per_launch": score_flops,
                     "executed_flops_per_launch": executed,
                     "executed_tflops": executed / (attn_ms * 1e-3) / 1e12 if executed else None,
                     "executed_frac": executed / (attn_ms * 1e-3) / 1e12 / peak if executed else None,
                     "useful_over_executed": attn_flops / executed if executed else None},
    }


def main_reference(args, w, info, rank, n_gpus):
    """Reference arm: the fp64 CPU oracle, timed as it stands, on rank 0 only."""
    if rank != 0:
        if info is not None:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return
    from block_sparse_long_15_b200 import workloads as W
    inp = W.make_inputs(w)
    per_step_s = max(1.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_oracle_rate(w, inp, per_step_s / 4, seed=1)
    rates = [cpu_oracle_rate(w, inp, per_step_s, seed=2 + i) for i in range(args.steps)]
    value = statistics.mean(r["value"] for r in rates)
    ms = 1e3 * real_rows(inp) / value
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": n_gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "ms_per_step_extrapolated": True,
           "ms_per_step_note": (f"extrapolated: the workload's {real_rows(inp)} real query rows divided by the "
                                "measured rows/s of the bounded samples; each timed step runs a sample only"),
           "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seq},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": rates[0]["cores"], "kind": "oracle",
                            "sample": f"each step: {rates[0]['sample']}"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    if info is not None:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
