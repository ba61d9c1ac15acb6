#!/usr/bin/env python
"""Benchmark of the compressed-KV hot path on B200.

One step = quantize-append of the new token's K/V (all KV heads) into the
compressed cache + split-K decode attention of every query head over the T
cached tokens, on the Llama-3.1-8B-shaped decode layer (B=1, 32 query / 8 KV
heads, d=128, T=32768, keys 3+QJL bits, values 4 bits, bf16 inputs, RoPE).
Prints ONE JSON line (rank 0).  Extra workloads (ESM-2-shaped prefill quantize
GB/s, long-context decode) are reported under "extras".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torch.distributed.run (one rank per GPU); every rank runs
its own independent replica of the workload (weak scaling, no collective on the
data path); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=200)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama_decode")
    p.add_argument("--no-extras", action="store_true")
    p.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--only", choices=["quantize_esm_prefill", "bidir_esm_prefill", "decode_long_context",
                                      "decode_llama", "vector_search", "quality", "decode_split",
                                      "decode_fibquant", "quality_fibquant", "haar"],
                   help="run one extra workload alone and print its JSON (1 GPU)")
    p.add_argument("--search-rows", type=int, default=0,
                   help="vector-search database rows for --only vector_search (default 10^6)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sust=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"], samples=0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9 and f[1].replace(".", "").isdigit():
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["no samples"], samples=0)
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=float(rows[0][2]), reasons=reasons,
                    samples=len(rows), power_w_max=max(float(r[3]) for r in rows
                                                        if r[3].replace(".", "").isdigit()))


def dist_init(backend: str = "nccl"):
    """Rank setup from the torchrun environment.  The process group carries
    only the barrier and the max-over-ranks timing (replicas share no data);
    ``backend="gloo"`` runs the same host logic on CPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput of N independent replicas: the units all ranks
    processed over the slowest rank's time."""
    return world * units_per_rank / max_seconds


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# Decode workload (quantize-append + split-K decode per step)
# ---------------------------------------------------------------------------

def row_bytes(w) -> int:
    """Compressed bytes per (token, KV head): key planes + (nu, rho), value planes + nu."""
    mse_k = w.bits_k - 1 if w.qjl_k else w.bits_k
    planes_k = mse_k + (1 if w.qjl_k else 0)
    return planes_k * w.d // 8 + 4 + w.bits_v * w.d // 8 + 2


def describe(w) -> str:
    mse_k = w.bits_k - 1 if w.qjl_k else w.bits_k
    kdesc = f"{mse_k}+QJL" if w.qjl_k else f"{mse_k}"
    rope = f" RoPE theta={w.rope_theta:g}" if w.rope_theta else ""
    return (f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} T={w.T} keys {kdesc} bits, "
            f"values {w.bits_v} bits, {w.dtype} inputs{rope}, "
            + (f"{w.num_splits} splits" if w.num_splits else "default split count"))


def haar_for(w):
    """Dense Haar rotation of a workload (library factorisation)."""
    from rotated_codebook_kv_tq_b200 import native, synth
    return native.haar_rotation(synth.haar_gaussian(w.d, w.seed))


class DecodeBench:
    def __init__(self, w, n_sets: int, haar: bool = False):
        import torch
        from rotated_codebook_kv_tq_b200 import native, synth
        self.w, self.n_sets = w, n_sets
        self.native = native
        D = synth.rotation_signs(w.d, w.seed)
        S = synth.qjl_matrix_bf16(w.d, w.seed) if w.qjl_k else None
        self.D, self.S = D, S
        self.codec = native.Codec(w.d, w.bits_k, w.qjl_k, w.bits_v, D, S,
                                  rotation=haar_for(w) if haar else None)
        T = w.T
        self.rows_cap = (T + 31) // 32 * 32
        K, V = synth.kv_inputs_torch(w, T=T)
        self.K, self.V = K, V
        r = synth.rope_for(w, self.rows_cap)
        self.rope_np = r
        self.rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
        self.caches = []
        for _ in range(n_sets):
            c = native.alloc_cache(self.codec, w.B, w.Hkv, self.rows_cap)
            native.quantize_kv(self.codec, K[:, :, :T - 1], V[:, :, :T - 1], c, row0=0,
                               rope=self.rope, pos0=0)
            self.caches.append(c)
        self.knew = K[:, :, T - 1:T].contiguous()
        self.vnew = V[:, :, T - 1:T].contiguous()
        self.q = synth.query_inputs_torch(w)[:, :, 0].contiguous()
        self.scale = 1.0 / math.sqrt(w.d)
        self.splits = w.num_splits
        nbytes = native.attention_workspace(self.codec, w.B, w.Hq, self.splits)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()

    def step(self, s: int, knew=None, vnew=None, q=None) -> None:
        """One decode step through tq_decode_step: append of the new token's
        K/V at row T - 1, then the decode of every query head over T rows."""
        w, n = self.w, self.native
        c = self.caches[s % self.n_sets]
        n.decode_step(self.codec, self.knew if knew is None else knew,
                      self.vnew if vnew is None else vnew, self.q if q is None else q, c, w.T,
                      self.scale, self.out, self.ws, rope=self.rope, num_splits=self.splits)

    def cache_bytes_per_step(self) -> int:
        return self.w.B * self.w.Hkv * self.w.T * row_bytes(self.w)


# Every TIMED_EVERY-th step of the timed graphs brackets its main-loop kernel
# with CUDA events.  An event node between two kernels turns their
# programmatic dependent launch into a full dependency, so bracketing every
# step would slow the steps being timed; sampling keeps that cost off the rest.
TIMED_EVERY = 10


def time_decode(bench: DecodeBench, K: int, W: int, world: int, sampler):
    """Warm up W steps, then time exactly K steps replayed from CUDA graphs.
    Returns (total seconds, mean chunk-kernel seconds, launches per step)."""
    import torch
    native = bench.native
    c0 = native.launch_count()
    bench.step(0)
    torch.cuda.synchronize()
    per_step = native.launch_count() - c0
    M = min(K, 250)
    n_ev = (M + TIMED_EVERY - 1) // TIMED_EVERY
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for ev in starts + stops:      # torch creates the CUDA event on first record
        ev.record()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(M):
            if i % TIMED_EVERY == 0:
                native.set_timing_events(starts[i // TIMED_EVERY], stops[i // TIMED_EVERY])
            bench.step(i)
            if i % TIMED_EVERY == 0:
                native.set_timing_events(None, None)
    rem = K % M
    tail = None
    if rem:
        tail = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tail):
            for i in range(rem):
                bench.step(i)
    for i in range(W):
        bench.step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.start()
    e0.record()
    for _ in range(K // M):
        graph.replay()
    if tail is not None:
        tail.replay()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    total = e0.elapsed_time(e1) / 1e3
    try:
        kern = statistics.mean(starts[i].elapsed_time(stops[i]) for i in range(n_ev)) / 1e3
    except Exception:
        # events in graphs unusable: bracket the kernel in direct launches instead
        kern = None
    del graph, tail
    if kern is None:
        sa, so = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for i in range(50):
            native.set_timing_events(sa, so)
            bench.step(i)
            native.set_timing_events(None, None)
            torch.cuda.synchronize()
            ts.append(sa.elapsed_time(so) / 1e3)
        kern = statistics.median(ts)
    return total, kern, per_step, clocks


def time_e2e(bench: DecodeBench, K: int, W: int):
    """Same step through the public API with host buffers: one tq_decode_step_host
    call per step copies the new token's K/V and the query from pinned host
    memory, runs the step and returns with the output in pinned host memory."""
    import torch
    native = bench.native
    # the step's inputs (new token's K and V, the query) packed in one pinned
    # host buffer, so each step is one host-to-device copy
    parts = (bench.knew, bench.vnew, bench.q)
    assert len({t.dtype for t in parts}) == 1
    hbuf = torch.cat([t.reshape(-1).cpu() for t in parts]).pin_memory()
    dbuf = torch.empty_like(hbuf, device=bench.q.device)
    oh = torch.empty(bench.out.shape, dtype=torch.float32).pin_memory()
    w = bench.w
    kvt, qt = bench.knew.dtype, bench.q.dtype

    def one(i):
        native.decode_step_host(bench.codec, hbuf, dbuf, kvt, qt, w.B, w.Hq, w.Hkv,
                                bench.caches[i % bench.n_sets], w.T, bench.scale, bench.out, oh,
                                bench.ws, rope=bench.rope, num_splits=bench.splits)

    for i in range(W):
        one(i)
    t0 = time.perf_counter()
    for i in range(K):
        one(i)
    dt = time.perf_counter() - t0
    h2d = hbuf.numel() * hbuf.element_size()
    d2h = oh.numel() * oh.element_size()
    return dt, h2d, d2h


# ---------------------------------------------------------------------------
# Oracle (CPU) baseline
# ---------------------------------------------------------------------------

class OracleDecode:
    """The CPU oracle run on the same workload: quantize-append of the new token,
    then estimator-form attention of every query head (fp64 numpy)."""

    def __init__(self, bench: DecodeBench):
        import numpy as np
        from oracle import codec as oc
        w = bench.w
        self.w, self.oc = w, oc
        self.codec = oc.make_codec(w.d, w.bits_k, w.qjl_k, w.bits_v, bench.D, bench.S)
        self.K = bench.K.float().cpu().numpy().astype(np.float64)
        self.V = bench.V.float().cpu().numpy().astype(np.float64)
        self.q = bench.q.float().cpu().numpy().astype(np.float64)
        self.rope = bench.rope_np
        self.rows_cap = bench.rows_cap
        self.cache = None

    def prefill(self, rows: int):
        """Untimed setup: cache rows 0 .. rows-2 (the new token is row rows-1)."""
        oc, w = self.oc, self.w
        self.n = rows
        self.cache = oc.empty_cache(self.codec, w.B, w.Hkv, (rows + 31) // 32 * 32)
        oc.quantize_into(self.cache, self.K[:, :, :rows - 1], self.V[:, :, :rows - 1], self.codec,
                         rope=self.rope)

    def step(self):
        from oracle import attention as oatt
        oc, w, n = self.oc, self.w, self.n
        oc.quantize_into(self.cache, self.K[:, :, n - 1:n], self.V[:, :, n - 1:n], self.codec,
                         rope=self.rope, pos0=n - 1, row0=n - 1)
        return oatt.decode(self.q, self.cache, self.codec, [n] * w.B, 1.0 / math.sqrt(w.d),
                           rope=self.rope)


def oracle_rate(bench: DecodeBench, seconds: float, rows: int = None):
    """Tokens/s of the oracle on a bounded sample: full decode steps over the
    first ``rows`` tokens of the context, scaled linearly to the full context
    (cost is linear in the number of cached tokens)."""
    w = bench.w
    rows = w.T if rows is None else rows
    o = OracleDecode(bench)
    o.prefill(rows)
    n, t0 = 0, time.perf_counter()
    while True:
        o.step()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or n >= 1000:
            break
    per_step_full = dt / n * (w.T / rows)
    return w.B / per_step_full, n, dt, rows


def _time_loop(fn, seconds: float) -> float:
    """Seconds per call of ``fn``: at least one call, then repeat until
    ``seconds`` have passed."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            return dt / n


def _one_and_all(fn, seconds: float):
    """(seconds per call on one thread, on every BLAS thread, thread count)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        t1 = _time_loop(fn, seconds)
    return t1, _time_loop(fn, seconds), blas_threads()


def cpu_baselines(seconds: float = 1.0) -> dict:
    """The oracle, as it stands, timed on this host on bounded samples of every
    workload, single-threaded and with all BLAS threads (numpy fp64; the Python
    loops over heads and rows stay on one core either way).  Each figure is in
    the unit of the matching GPU figure, scaled from the sample as stated."""
    import numpy as np
    from oracle import attention as oatt
    from oracle import codec as oc
    from oracle import scan as oscan
    from rotated_codebook_kv_tq_b200 import synth
    out = dict(nproc=os.cpu_count())

    def codec_of(w):
        S = synth.qjl_matrix_bf16(w.d, w.seed) if w.qjl_k else None
        return oc.make_codec(w.d, w.bits_k, w.qjl_k, w.bits_v, synth.rotation_signs(w.d, w.seed), S)

    def entry(unit, t1, tn, threads, to_value, sample):
        return dict(unit=unit, one_thread=to_value(t1), all_threads=to_value(tn), threads=threads,
                    sample=sample)

    # decode steps: quantize-append of the new token + attention of every head
    # over the first `rows` cached tokens; cost is linear in rows, scaled to T
    for name, rows in (("tiny", 1024), ("llama_decode", 1024), ("long_decode", 512)):
        w = synth.WORKLOADS[name]
        ww = w.scaled(T=rows)
        K, V = synth.kv_inputs(ww)
        q = synth.as_float64(synth.query_inputs(ww, Lq=1)[:, :, 0], w.dtype)
        K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
        codec = codec_of(w)
        rope = synth.rope_for(w, (rows + 31) // 32 * 32)
        cache = oc.empty_cache(codec, w.B, w.Hkv, (rows + 31) // 32 * 32)
        oc.quantize_into(cache, K64[:, :, :rows - 1], V64[:, :, :rows - 1], codec, rope=rope)

        def step():
            oc.quantize_into(cache, K64[:, :, rows - 1:], V64[:, :, rows - 1:], codec, rope=rope,
                             pos0=rows - 1, row0=rows - 1)
            oatt.decode(q, cache, codec, [rows] * w.B, 1.0 / math.sqrt(w.d), rope=rope)
        t1, tn, th = _one_and_all(step, seconds)
        scale = w.T / rows
        out[name] = entry("tokens/s", t1, tn, th, lambda t: w.B / (t * scale),
                          f"one decode step over the first {rows} of {w.T} tokens, all "
                          f"{w.B * w.Hq} query heads, time x {w.T}/{rows}")
    # the 2.5-bit outlier split on the Llama shape, same sampling as above
    from oracle import split as osp
    from oracle.rotation import apply_rope
    w = synth.WORKLOADS["llama_decode"]
    rows = 1024
    ww = w.scaled(T=rows)
    K, V = synth.kv_inputs(ww)
    K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
    q = synth.as_float64(synth.query_inputs(ww, Lq=1)[:, :, 0], w.dtype)
    rope = synth.rope_for(w, rows)
    halves = []
    for i, (bk, bv) in enumerate(SPLIT_RATES["2.5"]):
        ds, sd = w.d // 2, w.seed + 100 * (i + 1)
        halves.append(oc.make_codec(ds, bk, True, bv, synth.rotation_signs(ds, sd),
                                    synth.qjl_matrix_bf16(ds, sd)))
    Kr = np.stack([[apply_rope(K64[b, h], rope[0], rope[1], np.arange(rows)) for h in range(w.Hkv)]
                   for b in range(w.B)])
    score = np.stack([np.mean(Kr ** 2, axis=(0, 2)), np.mean(V64 ** 2, axis=(0, 2))], axis=1)
    sc = osp.make_split_codec(halves[0], halves[1], osp.outlier_channels(score))
    caches = osp.empty_caches(sc, w.B, w.Hkv, rows)
    osp.quantize_into(caches, K64[:, :, :rows - 1], V64[:, :, :rows - 1], sc, rope=rope)

    def split_step():
        osp.quantize_into(caches, K64[:, :, rows - 1:], V64[:, :, rows - 1:], sc, rope=rope,
                          pos0=rows - 1, row0=rows - 1)
        osp.decode(q, caches, sc, [rows] * w.B, 1.0 / math.sqrt(w.d), rope=rope)
    t1, tn, th = _one_and_all(split_step, seconds)
    out["decode_split_2.5bit"] = entry("tokens/s", t1, tn, th, lambda t: w.B / (t * w.T / rows),
                                       f"one split decode step over the first {rows} of {w.T} "
                                       f"tokens, all {w.B * w.Hq} query heads, time x {w.T}/{rows}")
    # FibQuant k = 2 at 2 bits per coordinate on the Llama shape, same sampling
    from oracle import fibquant as ofq
    fqc = ofq.make_codec(w.d, 4, 4, synth.rotation_signs(w.d, w.seed))
    fcache = ofq.empty_cache(fqc, w.B, w.Hkv, rows)
    ofq.quantize_into(fcache, K64[:, :, :rows - 1], V64[:, :, :rows - 1], fqc, rope=rope)

    def fq_step():
        ofq.quantize_into(fcache, K64[:, :, rows - 1:], V64[:, :, rows - 1:], fqc, rope=rope,
                          pos0=rows - 1, row0=rows - 1)
        ofq.decode(q, fcache, fqc, [rows] * w.B, 1.0 / math.sqrt(w.d), rope=rope)
    t1, tn, th = _one_and_all(fq_step, seconds)
    out["decode_fibquant_2bit"] = entry("tokens/s", t1, tn, th, lambda t: w.B / (t * w.T / rows),
                                        f"one FibQuant decode step over the first {rows} of {w.T} "
                                        f"tokens, all {w.B * w.Hq} query heads, time x {w.T}/{rows}")
    # ESM-2-shaped prefill quantize: two (batch, head) pairs of the 320
    w = synth.WORKLOADS["esm_prefill"]
    ww = w.scaled(B=1, Hq=2, Hkv=2)
    K, V = synth.kv_inputs(ww)
    K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
    codec = codec_of(w)
    rope = synth.rope_for(w, w.T)
    cache = oc.empty_cache(codec, 1, 2, w.T)
    t1, tn, th = _one_and_all(lambda: oc.quantize_into(cache, K64, V64, codec, rope=rope), seconds)
    in_bytes = 2 * 2 * w.T * w.d * 2
    out["quantize_esm_prefill"] = entry("GB/s of bf16 input", t1, tn, th, lambda t: in_bytes / t / 1e9,
                                        f"K+V of 2 of the {w.B * w.Hkv} (batch, head) pairs, T={w.T}")
    # ESM-2-shaped bidirectional pass: one head, all 1024 queries
    q = synth.as_float64(synth.query_inputs(ww, Lq=w.T), w.dtype)
    ropeq = synth.rope_for(w, w.T)
    flops = 2 * w.T * w.T * 2 * w.d + 2 * w.T * w.T * w.d
    t1, tn, th = _one_and_all(
        lambda: oatt.bidirectional(q, cache, codec, w.T, 1.0 / math.sqrt(w.d), rope=ropeq,
                                   heads=[(0, 0)]), seconds)
    out["bidir_esm_prefill"] = entry("TFLOP/s (algorithmic)", t1, tn, th, lambda t: flops / t / 1e12,
                                     f"one of the {w.B * w.Hq} heads, {w.T} queries x {w.T} keys")
    # vector search: index build of 2048 rows; scan of 8 queries over 8192 rows
    sw = synth.VECTOR_SEARCH
    scodec = oc.make_codec(sw.d, sw.bits, True, 4, synth.rotation_signs(sw.d, sw.seed),
                           synth.qjl_matrix_bf16(sw.d, sw.seed))
    x = synth.unit_rows(8192, sw.d, sw.seed, synth.STREAM_K).astype(np.float64)
    qs = synth.unit_rows(8, sw.d, sw.seed, synth.STREAM_Q).astype(np.float64)
    t1, tn, th = _one_and_all(lambda: oc.pack_keys(oc.quantize_keys(x[:2048], scodec), scodec), seconds)
    out["index_build"] = entry("rows/s", t1, tn, th, lambda t: 2048 / t, "2048 of the 10^6 rows")
    kc, ks = oc.pack_keys(oc.quantize_keys(x, scodec), scodec)
    t1, tn, th = _one_and_all(lambda: oscan.topk(oscan.scores(qs, kc, ks, scodec), sw.k), seconds)
    out["scan_topk"] = entry("queries/s over 10^6 rows", t1, tn, th,
                             lambda t: 8 * 8192 / t / sw.n, "8 queries x 8192 rows, scaled to 10^6 rows")
    return out


# ---------------------------------------------------------------------------
# Extra workloads
# ---------------------------------------------------------------------------

def quantize_extra(wname: str, pk: dict, steps: int = 40, haar: bool = False):
    """Prefill quantize of a whole [B, H, T, d] K/V batch: input GB/s and the
    kernel's HBM roofline fraction.  Rotates over input sets larger than L2.
    haar: the codec on a dense Haar rotation instead of the randomized WHT."""
    import torch
    from rotated_codebook_kv_tq_b200 import native, synth
    w = synth.WORKLOADS[wname]
    D = synth.rotation_signs(w.d, w.seed)
    S = synth.qjl_matrix_bf16(w.d, w.seed) if w.qjl_k else None
    codec = native.Codec(w.d, w.bits_k, w.qjl_k, w.bits_v, D, S,
                         rotation=haar_for(w) if haar else None)
    rows_cap = (w.T + 31) // 32 * 32
    in_bytes = 2 * w.B * w.Hkv * w.T * w.d * (2 if w.dtype == "bf16" else 4)
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    n_sets = max(2, math.ceil(3 * l2 / in_bytes))
    sets = []
    for s in range(n_sets):
        K, V = synth.kv_inputs_torch(w, seed_salt=s)
        sets.append((K, V, native.alloc_cache(codec, w.B, w.Hkv, rows_cap)))
    r = synth.rope_for(w, rows_cap)
    rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
    for K, V, c in sets:
        native.quantize_kv(codec, K, V, c, rope=rope)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        K, V, c = sets[i % n_sets]
        evs[i][0].record()
        native.quantize_kv(codec, K, V, c, rope=rope)
        evs[i][1].record()
    torch.cuda.synchronize()
    t = statistics.median(a.elapsed_time(b) for a, b in evs) / 1e3
    out_bytes = w.B * w.Hkv * w.T * row_bytes(w)
    alg = in_bytes + out_bytes
    return dict(workload=describe(w), rotation="dense Haar" if haar else "randomized WHT",
                input_GBps=in_bytes / t / 1e9, us_per_call=t * 1e6,
                roofline=dict(bound="hbm", achieved=alg / t / 1e9, peak=pk["hbm"], unit="GB/s",
                              frac=alg / t / 1e9 / pk["hbm"], algorithmic_bytes=alg),
                l2="rotating %d input sets (%.0f MB)" % (n_sets, n_sets * in_bytes / 1e6))


def _rope_rows(x, c, s):
    """Rotate-half RoPE of fp32 rows x [..., d] with cos/sin tables [..., d/2]."""
    import torch
    h = x.shape[-1] // 2
    u, v = x[..., :h], x[..., h:]
    return torch.cat((u * c - v * s, v * c + u * s), dim=-1)


def quality_extra(wname: str, T: int = 0, variants=("prod", "mse"), overrides=None):
    """Quality of the compressed cache on one workload, for the key codec with
    the 1-bit QJL residual sketch ("prod": TQ-QKV) and with the same key bits
    spent on the MSE stage alone ("mse": TQ-KV): relMSE_K and relMSE_V =
    sum ||x_hat - x||^2 / sum ||x||^2 over every cached row (x the post-RoPE
    key, the value as given, x_hat from tq_dequantize), and the cosine between
    each query head's compressed attention output (tq_attention_decode, or
    tq_attention_bidir for the bidirectional workload) and fp32 attention over
    the exact K/V, mean and minimum over heads (and queries)."""
    import torch
    from rotated_codebook_kv_tq_b200 import native, synth
    w = synth.WORKLOADS[wname]
    if T:
        w = w.scaled(T=T, Lq=min(w.Lq, T))
    if overrides:
        w = w.scaled(**overrides)
    rows_cap = (w.T + 31) // 32 * 32
    K, V = synth.kv_inputs_torch(w)
    bidir = w.Lq > 1
    q = synth.query_inputs_torch(w, Lq=w.Lq if bidir else 1)
    r = synth.rope_for(w, max(rows_cap, w.Lq))
    rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
    Kf, Vf, qf = K.float(), V.float(), q.float()
    if rope is not None:
        Kf = _rope_rows(Kf, rope[0][:w.T], rope[1][:w.T])
        if bidir:
            qf = _rope_rows(qf, rope[0][:w.Lq], rope[1][:w.Lq])
        else:
            qf = _rope_rows(qf, rope[0][w.T - 1], rope[1][w.T - 1])
    scale = 1.0 / math.sqrt(w.d)
    # exact attention, fp32, GQA: query head h reads KV head h // G
    Ke = Kf.repeat_interleave(w.G, dim=1)
    Ve = Vf.repeat_interleave(w.G, dim=1)
    p = torch.softmax(torch.matmul(qf, Ke.transpose(-1, -2)) * scale, dim=-1)
    o_ref = torch.matmul(p, Ve)                       # [B, Hq, Lq, d]
    del Ke, Ve, p
    D = synth.rotation_signs(w.d, w.seed)
    S = synth.qjl_matrix_bf16(w.d, w.seed)
    out = {}
    for var in variants:
        qjl = var == "prod"
        codec = native.Codec(w.d, w.bits_k, qjl, w.bits_v, D, S if qjl else None)
        cache = native.alloc_cache(codec, w.B, w.Hkv, rows_cap)
        native.quantize_kv(codec, K, V, cache, rope=rope)
        rel = {}
        for which, x in ((0, Kf), (1, Vf)):
            xh = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.float32, device="cuda")
            native.dequantize(codec, cache, which, 0, w.T, xh)
            rel["K" if which == 0 else "V"] = float(((xh - x) ** 2).sum() / (x ** 2).sum())
            del xh
        res = dict(key_bits=w.bits_k, key_mse_bits=w.bits_k - 1 if qjl else w.bits_k,
                   value_bits=w.bits_v, relMSE_K=rel["K"], relMSE_V=rel["V"])
        try:
            if bidir:
                o = torch.empty((w.B, w.Hq, w.Lq, w.d), dtype=torch.float32, device="cuda")
                ws = torch.empty(native.attention_bidir_workspace(codec, w.B, w.Hq, w.Lq),
                                 dtype=torch.uint8, device="cuda")
                native.attention_bidir(codec, q, cache, w.T, scale, o, ws, rope=rope)
            else:
                o = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
                ws = torch.empty(native.attention_workspace(codec, w.B, w.Hq, w.num_splits),
                                 dtype=torch.uint8, device="cuda")
                native.attention_decode(codec, q[:, :, 0], cache, w.T, scale, o, ws, rope=rope,
                                        num_splits=w.num_splits)
                o = o[:, :, None]
            cos = torch.nn.functional.cosine_similarity(o, o_ref, dim=-1)
            res.update(output_cosine_mean=float(cos.mean()), output_cosine_min=float(cos.min()))
        except native.TqError as e:
            res.update(output_cosine_mean=None, output_cosine_min=None, attention=str(e))
        out[var] = res
        del cache
        codec.close()
    torch.cuda.synchronize()
    return dict(workload=describe(w), variants=out,
                definition="relMSE = sum||x_hat-x||^2/sum||x||^2 over all rows (K post-RoPE); "
                           "cosine of each head's output vs fp32 attention over exact K/V")


def bidir_extra(pk: dict, steps: int = 10):
    """ESM-2-shaped bidirectional pass over the compressed cache (every query
    attends to every key): algorithmic flops 2 T^2 (2d) + 2 T^2 d per head
    (logits from the rotated MSE + QJL columns, then P V)."""
    import torch
    from rotated_codebook_kv_tq_b200 import native, synth
    w = synth.WORKLOADS["esm_prefill"]
    D = synth.rotation_signs(w.d, w.seed)
    S = synth.qjl_matrix_bf16(w.d, w.seed)
    codec = native.Codec(w.d, w.bits_k, w.qjl_k, w.bits_v, D, S)
    rows_cap = (w.T + 31) // 32 * 32
    r = synth.rope_for(w, max(rows_cap, w.Lq))
    rope = (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
    K, V = synth.kv_inputs_torch(w)
    cache = native.alloc_cache(codec, w.B, w.Hkv, rows_cap)
    native.quantize_kv(codec, K, V, cache, rope=rope)
    q = synth.query_inputs_torch(w, Lq=w.Lq)
    out = torch.empty((w.B, w.Hq, w.Lq, w.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(native.attention_bidir_workspace(codec, w.B, w.Hq, w.Lq), dtype=torch.uint8,
                     device="cuda")
    scale = 1.0 / math.sqrt(w.d)
    sa, so = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for ev in (sa, so, e0, e1):      # torch creates the CUDA event on first record
        ev.record()
    for _ in range(2):
        native.attention_bidir(codec, q, cache, w.T, scale, out, ws, rope=rope)
    torch.cuda.synchronize()
    kt, tt = [], []
    for _ in range(steps):
        native.set_timing_events(sa, so)
        e0.record()
        native.attention_bidir(codec, q, cache, w.T, scale, out, ws, rope=rope)
        e1.record()
        native.set_timing_events(None, None)
        torch.cuda.synchronize()
        kt.append(sa.elapsed_time(so) / 1e3)
        tt.append(e0.elapsed_time(e1) / 1e3)
    flops = w.B * w.Hq * (2 * w.T * w.Lq * 2 * w.d + 2 * w.T * w.Lq * w.d)
    k = statistics.median(kt)
    return dict(workload=describe(w) + f", Lq={w.Lq} bidirectional", us_per_call=statistics.median(tt) * 1e6,
                roofline=dict(bound="tensor", achieved=flops / k / 1e12, peak=pk["bf16"], unit="TFLOP/s",
                              frac=flops / k / 1e12 / pk["bf16"], algorithmic_flops=flops,
                              kernel="bidir_tile_kernel", kernel_us=k * 1e6,
                              note="three-term bf16 split: 6 MMA sets per product, not counted in flops"))


def search_extra(pk: dict, steps: int = 5):
    """Vector search, d = 1536, TurboQuant_prod at 4 bits: index build of 10^6
    unit rows (input fp32 GB/s; the QJL sketch is 2 d^2 flops per row on the
    tensor cores) and the inner-product scan + top-10 of 1024 queries
    (2 * 3072 flops per (row, query), the estimator as one GEMM)."""
    import torch
    from rotated_codebook_kv_tq_b200 import native, synth
    w = synth.VECTOR_SEARCH
    codec = native.Codec(w.d, w.bits, True, 4, synth.rotation_signs(w.d, w.seed),
                         synth.qjl_matrix_bf16(w.d, w.seed))
    g = torch.Generator(device="cuda")
    g.manual_seed(w.seed * 1000)
    x = torch.randn((w.n, w.d), generator=g, device="cuda")
    x /= x.norm(dim=1, keepdim=True)
    q = torch.randn((w.nq, w.d), generator=g, device="cuda")
    q /= q.norm(dim=1, keepdim=True)
    kcode = torch.empty((w.n, codec.planes_k, w.d // 8), dtype=torch.uint8, device="cuda")
    kscale = torch.empty((w.n, 2), dtype=torch.float16, device="cuda")
    iws = torch.empty(native.index_workspace(codec, w.n), dtype=torch.uint8, device="cuda")
    idx = torch.empty((w.nq, w.k), dtype=torch.int32, device="cuda")
    score = torch.empty((w.nq, w.k), dtype=torch.float32, device="cuda")
    sws = torch.empty(native.scan_workspace(codec, w.n, w.nq, w.k), dtype=torch.uint8, device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record()
    native.index_build(codec, x, kcode, kscale, iws)
    native.scan_topk(codec, kcode, kscale, q, w.k, idx, score, sws)
    torch.cuda.synchronize()
    bt, st, kt = [], [], []
    for _ in range(steps):
        ev[0].record()
        native.index_build(codec, x, kcode, kscale, iws)
        ev[1].record()
        native.set_timing_events(ev[2], ev[3])
        e_s0, e_s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_s0.record()
        native.scan_topk(codec, kcode, kscale, q, w.k, idx, score, sws)
        e_s1.record()
        native.set_timing_events(None, None)
        torch.cuda.synchronize()
        bt.append(ev[0].elapsed_time(ev[1]) / 1e3)
        st.append(e_s0.elapsed_time(e_s1) / 1e3)
        kt.append(ev[2].elapsed_time(ev[3]) / 1e3)
    b, s_, k = statistics.median(bt), statistics.median(st), statistics.median(kt)
    # the lookup-table scan (fp32 scores) on the first 64 queries, for comparison
    nql = 64
    ql = q[:nql].contiguous()
    il = torch.empty((nql, w.k), dtype=torch.int32, device="cuda")
    sl = torch.empty((nql, w.k), dtype=torch.float32, device="cuda")
    native.scan_topk_lut(codec, kcode, kscale, ql, w.k, il, sl, sws)
    torch.cuda.synchronize()
    e_l0, e_l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_l0.record()
    native.scan_topk_lut(codec, kcode, kscale, ql, w.k, il, sl, sws)
    e_l1.record()
    torch.cuda.synchronize()
    lt = e_l0.elapsed_time(e_l1) / 1e3
    in_bytes = w.n * w.d * 4
    sketch_flops = 2 * w.n * w.d * w.d
    scan_flops = 2 * 2 * w.d * w.n * w.nq
    return dict(
        workload=f"vector_search: n={w.n} d={w.d} fp32 unit rows, nq={w.nq}, TurboQuant_prod "
                 f"{w.bits} bits, top-{w.k}",
        index_build=dict(ms_per_call=b * 1e3, input_GBps=in_bytes / b / 1e9,
                         rows_per_s=w.n / b,
                         roofline=dict(bound="tensor", achieved=sketch_flops / b / 1e12,
                                       peak=pk["bf16"], unit="TFLOP/s",
                                       frac=sketch_flops / b / 1e12 / pk["bf16"],
                                       algorithmic_flops=sketch_flops,
                                       note="whole call (encode + sketch GEMM); bf16 hi/lo split: "
                                            "2 MMA passes, not counted")),
        scan_topk=dict(ms_per_call=s_ * 1e3, queries_per_s=w.nq / s_,
                       roofline=dict(bound="tensor", achieved=scan_flops / k / 1e12, peak=pk["bf16"],
                                     unit="TFLOP/s", frac=scan_flops / k / 1e12 / pk["bf16"],
                                     algorithmic_flops=scan_flops, kernel="ix_scan2_kernel",
                                     kernel_ms=k * 1e3)),
        scan_topk_lut=dict(queries=nql, ms_per_call=lt * 1e3, queries_per_s=nql / lt,
                           note="lookup-table scan, fp32 scores, same database; the comparison "
                                "path to the tensor-core scan"),
        l2="database codes 772 MB and input 6.1 GB > L2")


def decode_extra(wname: str, pk: dict, steps: int = 60, warmup: int = 5, haar: bool = False,
                 n_sets: int = 1):
    import torch
    from rotated_codebook_kv_tq_b200 import synth
    w = synth.WORKLOADS[wname]
    bench = DecodeBench(w, n_sets=n_sets, haar=haar)

    class _Null:
        def start(self):
            pass

        def stop(self):
            return {}

    total, kern, _, _ = time_decode(bench, steps, warmup, 1, _Null())
    alg = bench.cache_bytes_per_step()
    res = dict(workload=describe(w), rotation="dense Haar" if haar else "randomized WHT",
               us_per_step=total / steps * 1e6, tokens_per_s=w.B * steps / total,
               roofline=dict(bound="hbm", achieved=alg / kern / 1e9, peak=pk["hbm"], unit="GB/s",
                             frac=alg / kern / 1e9 / pk["hbm"], algorithmic_bytes=alg,
                             kernel_us=kern * 1e6),
               l2="rotating %d cache(s) of %.0f MB" % (n_sets, alg / 1e6))
    del bench
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# Outlier-channel split ("Google presenta TurboQuant ...", "Desempeno teorico y
# empirico": outlier channels at more bits than the rest)
# ---------------------------------------------------------------------------

SPLIT_RATES = {"2.5": ((3, 3), (2, 2)), "3.5": ((4, 4), (3, 3))}


def split_codecs(w, rate: str):
    """(hi, lo) library codecs of d/2 channels each, QJL keys: ``rate`` bits per
    channel as the mean of the two codecs' widths."""
    from rotated_codebook_kv_tq_b200 import native, synth
    out = []
    for i, (bk, bv) in enumerate(SPLIT_RATES[rate]):
        ds, seed = w.d // 2, w.seed + 100 * (i + 1)
        out.append(native.Codec(ds, bk, True, bv, synth.rotation_signs(ds, seed),
                                synth.qjl_matrix_bf16(ds, seed)))
    return out


def split_row_bytes(hi, lo) -> int:
    return sum(c.planes_k * c.d // 8 + 4 + c.bits_v * c.d // 8 + 2 for c in (hi, lo))


def split_channel_lists(Kr, V):
    """Per KV head: keys' and values' d/2 highest mean-square channels (keys
    after RoPE, as the codec sees them) -> device int16 [Hkv, 2, d]."""
    import torch
    from rotated_codebook_kv_tq_b200 import native
    score = torch.stack([(Kr.float() ** 2).mean(dim=(0, 2)), (V.float() ** 2).mean(dim=(0, 2))], dim=1)
    return torch.from_numpy(native.split_channels(score.cpu().numpy())).cuda()


class SplitBench:
    """Decode step over the split cache: quantize-append of the new token into
    both caches, then tq_attention_decode_split (same interface as DecodeBench
    for time_decode)."""

    def __init__(self, w, rate: str, n_sets: int):
        import torch
        from rotated_codebook_kv_tq_b200 import native, synth
        self.w, self.native, self.n_sets = w, native, n_sets
        hi, lo = split_codecs(w, rate)
        T = w.T
        self.rows_cap = (T + 31) // 32 * 32
        K, V = synth.kv_inputs_torch(w, T=T)
        r = synth.rope_for(w, self.rows_cap)
        self.rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
        Kr = K.float() if self.rope is None else _rope_rows(K.float(), self.rope[0][:T], self.rope[1][:T])
        self.split = native.Split(hi, lo, split_channel_lists(Kr, V))
        del Kr
        self.caches = []
        for _ in range(n_sets):
            ch = native.alloc_cache(hi, w.B, w.Hkv, self.rows_cap)
            cl = native.alloc_cache(lo, w.B, w.Hkv, self.rows_cap)
            native.quantize_kv_split(self.split, K[:, :, :T - 1], V[:, :, :T - 1], ch, cl,
                                     rope=self.rope)
            self.caches.append((ch, cl))
        self.knew = K[:, :, T - 1:T].contiguous()
        self.vnew = V[:, :, T - 1:T].contiguous()
        self.q = synth.query_inputs_torch(w)[:, :, 0].contiguous()
        self.scale = 1.0 / math.sqrt(w.d)
        self.splits = w.num_splits
        self.ws = torch.empty(native.attention_split_workspace(self.split, w.B, w.Hq, self.splits),
                              dtype=torch.uint8, device="cuda")
        self.out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        self.row_bytes = split_row_bytes(hi, lo)
        torch.cuda.synchronize()

    def step(self, s: int) -> None:
        w, n = self.w, self.native
        ch, cl = self.caches[s % self.n_sets]
        n.quantize_kv_split(self.split, self.knew, self.vnew, ch, cl, row0=w.T - 1, rope=self.rope,
                            pos0=w.T - 1)
        n.attention_decode_split(self.split, self.q, ch, cl, w.T, self.scale, self.out, self.ws,
                                 rope=self.rope, num_splits=self.splits)

    def cache_bytes_per_step(self) -> int:
        return self.w.B * self.w.Hkv * self.w.T * self.row_bytes


def split_decode_extra(pk: dict, rate: str = "2.5", steps: int = 40, warmup: int = 5):
    """Llama-shaped decode over the outlier-channel split cache (CUDA-core
    split-K kernels): tokens/s and the chunk kernel's HBM roofline fraction."""
    import torch
    from rotated_codebook_kv_tq_b200 import synth
    w = synth.WORKLOADS["llama_decode"]
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    hi, lo = split_codecs(w, rate)
    per_set = w.B * w.Hkv * ((w.T + 31) // 32 * 32) * split_row_bytes(hi, lo)
    hi.close()
    lo.close()
    bench = SplitBench(w, rate, max(1, math.ceil(3 * l2 / per_set)))

    class _Null:
        def start(self):
            pass

        def stop(self):
            return {}

    total, kern, per_step, _ = time_decode(bench, steps, warmup, 1, _Null())
    alg = bench.cache_bytes_per_step()
    res = dict(workload=f"llama_decode split {rate} bits per channel: B={w.B} Hq={w.Hq} "
                        f"Hkv={w.Hkv} d={w.d} T={w.T}, outlier halves {SPLIT_RATES[rate]} "
                        "(keys incl. QJL, values), per-head channel lists from the prefill",
               us_per_step=total / steps * 1e6, tokens_per_s=w.B * steps / total,
               launches_per_step=per_step,
               roofline=dict(bound="hbm", achieved=alg / kern / 1e9, peak=pk["hbm"], unit="GB/s",
                             frac=alg / kern / 1e9 / pk["hbm"], algorithmic_bytes=alg,
                             bytes_per_token_head=bench.row_bytes, kernel="split_chunk_kernel",
                             kernel_us=kern * 1e6),
               l2=f"rotating {bench.n_sets} split caches ({bench.n_sets * alg / 1e6:.0f} MB)")
    del bench
    torch.cuda.empty_cache()
    return res


def split_quality_extra(wname: str = "llama_decode"):
    """relMSE_K, relMSE_V and attention-output cosine (definitions as in
    quality_extra) of the 2.5- and 3.5-bit outlier splits, beside uniform
    codecs of 2, 3 and 4 bits (keys with QJL) on the same inputs."""
    import torch
    from rotated_codebook_kv_tq_b200 import native, synth
    w = synth.WORKLOADS[wname]
    rows_cap = (w.T + 31) // 32 * 32
    K, V = synth.kv_inputs_torch(w)
    q = synth.query_inputs_torch(w, Lq=1)[:, :, 0].contiguous()
    r = synth.rope_for(w, rows_cap)
    rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
    Kf, Vf, qf = K.float(), V.float(), q.float()
    if rope is not None:
        Kf = _rope_rows(Kf, rope[0][:w.T], rope[1][:w.T])
        qf = _rope_rows(qf, rope[0][w.T - 1], rope[1][w.T - 1])
    scale = 1.0 / math.sqrt(w.d)
    Ke = Kf.repeat_interleave(w.G, dim=1)
    Ve = Vf.repeat_interleave(w.G, dim=1)
    p = torch.softmax(torch.einsum("bhd,bhtd->bht", qf, Ke) * scale, dim=-1)
    o_ref = torch.einsum("bht,bhtd->bhd", p, Ve)
    del Ke, Ve, p
    chan = split_channel_lists(Kf, Vf)

    def scores(deq, decode):
        rel = {}
        for which, x in ((0, Kf), (1, Vf)):
            xh = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.float32, device="cuda")
            deq(which, xh)
            rel["K" if which == 0 else "V"] = float(((xh - x) ** 2).sum() / (x ** 2).sum())
            del xh
        o = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        decode(o)
        cos = torch.nn.functional.cosine_similarity(o, o_ref, dim=-1)
        return dict(relMSE_K=rel["K"], relMSE_V=rel["V"], output_cosine_mean=float(cos.mean()),
                    output_cosine_min=float(cos.min()))

    out = {}
    for rate in SPLIT_RATES:
        hi, lo = split_codecs(w, rate)
        sp = native.Split(hi, lo, chan)
        ch = native.alloc_cache(hi, w.B, w.Hkv, rows_cap)
        cl = native.alloc_cache(lo, w.B, w.Hkv, rows_cap)
        native.quantize_kv_split(sp, K, V, ch, cl, rope=rope)
        ws = torch.empty(native.attention_split_workspace(sp, w.B, w.Hq, w.num_splits),
                         dtype=torch.uint8, device="cuda")
        out[f"split_{rate}"] = dict(
            bits_per_channel=float(rate), halves=SPLIT_RATES[rate],
            **scores(lambda which, xh: native.dequantize_split(sp, ch, cl, which, 0, w.T, xh),
                     lambda o: native.attention_decode_split(sp, q, ch, cl, w.T, scale, o, ws,
                                                             rope=rope, num_splits=w.num_splits)))
        del ch, cl
        hi.close()
        lo.close()
    for bits in (2, 3, 4):
        D = synth.rotation_signs(w.d, w.seed)
        S = synth.qjl_matrix_bf16(w.d, w.seed)
        codec = native.Codec(w.d, bits, True, bits, D, S)
        cache = native.alloc_cache(codec, w.B, w.Hkv, rows_cap)
        native.quantize_kv(codec, K, V, cache, rope=rope)
        ws = torch.empty(native.attention_workspace(codec, w.B, w.Hq, w.num_splits),
                         dtype=torch.uint8, device="cuda")
        out[f"uniform_{bits}"] = dict(
            bits_per_channel=float(bits),
            **scores(lambda which, xh: native.dequantize(codec, cache, which, 0, w.T, xh),
                     lambda o: native.attention_decode(codec, q, cache, w.T, scale, o, ws,
                                                       rope=rope, num_splits=w.num_splits)))
        del cache
        codec.close()
    torch.cuda.synchronize()
    return dict(workload=describe(w), rows=out,
                channels="per KV head, the d/2 highest mean-square channels of the keys (after "
                         "RoPE) and of the values over the whole prefill")


# ---------------------------------------------------------------------------
# FibQuant k = 2 ("FibQuant ...", sections 2.1-2.3: a shared code for pairs of
# rotated coordinates, rate log2(N)/2 bits per coordinate)
# ---------------------------------------------------------------------------

def fq_row_bytes(codec) -> int:
    return codec.bits_k * codec.d // 16 + 4 + codec.bits_v * codec.d // 16 + 2


class FqBench:
    """Decode step with the FibQuant codec: quantize-append of the new token,
    then tq_fq_attention_decode (same interface as DecodeBench for time_decode)."""

    def __init__(self, w, bits: int, n_sets: int):
        import torch
        from rotated_codebook_kv_tq_b200 import native, synth
        self.w, self.native, self.n_sets = w, native, n_sets
        self.codec = native.FqCodec(w.d, bits, bits, synth.rotation_signs(w.d, w.seed))
        T = w.T
        self.rows_cap = (T + 31) // 32 * 32
        K, V = synth.kv_inputs_torch(w, T=T)
        r = synth.rope_for(w, self.rows_cap)
        self.rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
        self.caches = []
        for _ in range(n_sets):
            c = native.fq_alloc_cache(self.codec, w.B, w.Hkv, self.rows_cap)
            native.fq_quantize_kv(self.codec, K[:, :, :T - 1], V[:, :, :T - 1], c, rope=self.rope)
            self.caches.append(c)
        self.knew = K[:, :, T - 1:T].contiguous()
        self.vnew = V[:, :, T - 1:T].contiguous()
        self.q = synth.query_inputs_torch(w)[:, :, 0].contiguous()
        self.scale = 1.0 / math.sqrt(w.d)
        self.splits = w.num_splits
        self.ws = torch.empty(native.fq_attention_workspace(self.codec, w.B, w.Hq, self.splits),
                              dtype=torch.uint8, device="cuda")
        self.out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        self.row_bytes = fq_row_bytes(self.codec)
        torch.cuda.synchronize()

    def step(self, s: int) -> None:
        w, n = self.w, self.native
        c = self.caches[s % self.n_sets]
        n.fq_quantize_kv(self.codec, self.knew, self.vnew, c, row0=w.T - 1, rope=self.rope,
                         pos0=w.T - 1)
        n.fq_attention_decode(self.codec, self.q, c, w.T, self.scale, self.out, self.ws,
                              rope=self.rope, num_splits=self.splits)

    def cache_bytes_per_step(self) -> int:
        return self.w.B * self.w.Hkv * self.w.T * self.row_bytes


def fq_decode_extra(pk: dict, bits: int = 4, steps: int = 40, warmup: int = 5):
    """Llama-shaped decode over a FibQuant cache (bits per pair for keys and
    values; bits/2 per coordinate): tokens/s and the chunk kernel's roofline."""
    import torch
    from rotated_codebook_kv_tq_b200 import synth
    w = synth.WORKLOADS["llama_decode"]
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    per_set = w.B * w.Hkv * ((w.T + 31) // 32 * 32) * (2 * bits * w.d // 16 + 6)
    bench = FqBench(w, bits, max(1, math.ceil(3 * l2 / per_set)))

    class _Null:
        def start(self):
            pass

        def stop(self):
            return {}

    total, kern, per_step, _ = time_decode(bench, steps, warmup, 1, _Null())
    alg = bench.cache_bytes_per_step()
    res = dict(workload=f"llama_decode with FibQuant k=2, {bits} bits per pair ({bits / 2:g} per "
                        f"coordinate) for keys and values: B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} "
                        f"T={w.T}",
               us_per_step=total / steps * 1e6, tokens_per_s=w.B * steps / total,
               launches_per_step=per_step,
               roofline=dict(bound="hbm", achieved=alg / kern / 1e9, peak=pk["hbm"], unit="GB/s",
                             frac=alg / kern / 1e9 / pk["hbm"], algorithmic_bytes=alg,
                             bytes_per_token_head=bench.row_bytes, kernel="fq_chunk_kernel",
                             kernel_us=kern * 1e6),
               l2=f"rotating {bench.n_sets} caches ({bench.n_sets * alg / 1e6:.0f} MB)")
    del bench
    torch.cuda.empty_cache()
    return res


def fq_quality_extra(wname: str = "llama_decode", overrides=None):
    """relMSE_K, relMSE_V and output cosine (as in quality_extra) of FibQuant
    k = 2 at 0.5 .. 3 bits per coordinate beside the scalar MSE-only codec
    (TQ-KV) at 1, 2 and 3 bits, on the same inputs."""
    import torch
    from rotated_codebook_kv_tq_b200 import native, synth
    w = synth.WORKLOADS[wname]
    if overrides:
        w = w.scaled(**overrides)
    rows_cap = (w.T + 31) // 32 * 32
    K, V = synth.kv_inputs_torch(w)
    q = synth.query_inputs_torch(w, Lq=1)[:, :, 0].contiguous()
    r = synth.rope_for(w, rows_cap)
    rope = None if r is None else (torch.from_numpy(r[0]).cuda(), torch.from_numpy(r[1]).cuda())
    Kf, Vf, qf = K.float(), V.float(), q.float()
    if rope is not None:
        Kf = _rope_rows(Kf, rope[0][:w.T], rope[1][:w.T])
        qf = _rope_rows(qf, rope[0][w.T - 1], rope[1][w.T - 1])
    scale = 1.0 / math.sqrt(w.d)
    Ke = Kf.repeat_interleave(w.G, dim=1)
    Ve = Vf.repeat_interleave(w.G, dim=1)
    p = torch.softmax(torch.einsum("bhd,bhtd->bht", qf, Ke) * scale, dim=-1)
    o_ref = torch.einsum("bht,bhtd->bhd", p, Ve)
    del Ke, Ve, p
    D = synth.rotation_signs(w.d, w.seed)

    def scores(deq, decode):
        rel = {}
        for which, x in ((0, Kf), (1, Vf)):
            xh = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.float32, device="cuda")
            deq(which, xh)
            rel["K" if which == 0 else "V"] = float(((xh - x) ** 2).sum() / (x ** 2).sum())
            del xh
        o = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        decode(o)
        cos = torch.nn.functional.cosine_similarity(o, o_ref, dim=-1)
        return dict(relMSE_K=rel["K"], relMSE_V=rel["V"], output_cosine_mean=float(cos.mean()),
                    output_cosine_min=float(cos.min()))

    out = {}
    for bits in (1, 2, 3, 4, 5, 6):
        c = native.FqCodec(w.d, bits, bits, D)
        cache = native.fq_alloc_cache(c, w.B, w.Hkv, rows_cap)
        native.fq_quantize_kv(c, K, V, cache, rope=rope)
        ws = torch.empty(native.fq_attention_workspace(c, w.B, w.Hq, w.num_splits), dtype=torch.uint8,
                         device="cuda")
        out[f"fibquant_{bits / 2:g}"] = dict(
            bits_per_coordinate=bits / 2,
            **scores(lambda which, xh: native.fq_dequantize(c, cache, which, 0, w.T, xh),
                     lambda o: native.fq_attention_decode(c, q, cache, w.T, scale, o, ws, rope=rope,
                                                          num_splits=w.num_splits)))
        del cache
        c.close()
    for bits in (1, 2, 3):
        c = native.Codec(w.d, bits, False, bits, D, None)
        cache = native.alloc_cache(c, w.B, w.Hkv, rows_cap)
        native.quantize_kv(c, K, V, cache, rope=rope)
        ws = torch.empty(native.attention_workspace(c, w.B, w.Hq, w.num_splits), dtype=torch.uint8,
                         device="cuda")
        out[f"scalar_{bits}"] = dict(
            bits_per_coordinate=float(bits),
            **scores(lambda which, xh: native.dequantize(c, cache, which, 0, w.T, xh),
                     lambda o: native.attention_decode(c, q, cache, w.T, scale, o, ws, rope=rope,
                                                       num_splits=w.num_splits)))
        del cache
        c.close()
    torch.cuda.synchronize()
    return dict(workload=describe(w), rows=out,
                note="FibQuant keys and values both use the pair code (no QJL); scalar rows are "
                     "the MSE-only key codec (TQ-KV) at the same bits for keys and values")


def ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of ``kernel`` from the committed ncu summary, or
    None when the kernel's source changed after the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(kernel)
    if not d:
        return None
    src = os.path.join(ROOT, "rotated_codebook_kv_tq_b200", "csrc", d["source"])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] if os.path.exists(src) else None
    return d["bytes_per_launch"] if h == d.get("source_sha") else None


# ---------------------------------------------------------------------------
# Reference arm: the CPU oracle, timed on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import numpy as np
    from rotated_codebook_kv_tq_b200 import synth
    w = synth.WORKLOADS[args.workload]
    budget = 150.0
    steps = args.steps + args.warmup

    def oracle_for(rows):
        ww = w.scaled(T=rows)
        K, V = synth.kv_inputs(ww)
        q = synth.query_inputs(ww, Lq=1)[:, :, 0]
        o = OracleDecode.__new__(OracleDecode)
        from oracle import codec as oc
        o.w, o.oc = w, oc
        S = synth.qjl_matrix_bf16(w.d, w.seed) if w.qjl_k else None
        o.codec = oc.make_codec(w.d, w.bits_k, w.qjl_k, w.bits_v, synth.rotation_signs(w.d, w.seed), S)
        o.K, o.V = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
        o.q = synth.as_float64(q, w.dtype)
        o.rope = synth.rope_for(w, (rows + 31) // 32 * 32)
        o.prefill(rows)
        return o

    probe = oracle_for(256)
    t0 = time.perf_counter()
    for _ in range(3):
        probe.step()
    t256 = (time.perf_counter() - t0) / 3
    # cost ~ a + b * rows; take the probe as the per-step floor and size rows
    per_step_budget = budget / steps
    rows = int(max(32, min(w.T, 256 * per_step_budget / max(t256, 1e-9))))
    rows = rows // 32 * 32 or 32
    o = probe if rows == 256 else oracle_for(rows)
    for _ in range(args.warmup):
        o.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.step()
    dt = time.perf_counter() - t0
    per_step_full = dt / args.steps * (w.T / rows)
    value = w.B / per_step_full
    cores = blas_threads()
    sample = (f"each step: oracle quantize-append + decode of all {w.Hq} query heads over the "
              f"first {rows} of {w.T} cached tokens, time scaled by {w.T}/{rows}")
    line = dict(impl="reference", metric="compressed-KV decode tokens/s", value=value,
                unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=per_step_full * 1e3, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(workload=describe(w)),
                cpu_baseline=dict(value=value, unit="tokens/s", cores=cores, kind="oracle",
                                  sample=sample),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# Main
# ---------------------------------------------------------------------------

def smi_index(local: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


def run_only(args) -> int:
    """One extra workload on its own (profiling entry point)."""
    from rotated_codebook_kv_tq_b200.build import build
    build()
    pk = peaks()
    if args.only == "quantize_esm_prefill":
        r = quantize_extra("esm_prefill", pk, steps=3)
    elif args.only == "bidir_esm_prefill":
        r = bidir_extra(pk, steps=1)
    elif args.only == "decode_long_context":
        r = decode_extra("long_decode", pk, steps=5, warmup=3)
    elif args.only == "decode_llama":
        r = decode_extra("llama_decode", pk, steps=5, warmup=3)
    elif args.only == "quality":
        r = {name: quality_extra(name) for name in ("tiny", "llama_decode", "esm_prefill", "long_decode")}
        r["llama_decode_without_outliers"] = quality_extra(
            "llama_decode", overrides=dict(n_outliers=0, sigma_scale=None))
        r["llama_decode_outlier_split"] = split_quality_extra("llama_decode")
    elif args.only == "decode_split":
        r = {rate: split_decode_extra(pk, rate) for rate in SPLIT_RATES}
    elif args.only == "haar":
        r = dict(decode_llama=decode_extra("llama_decode", pk, steps=40, haar=True, n_sets=12),
                 decode_llama_wht=decode_extra("llama_decode", pk, steps=40, n_sets=12),
                 quantize_esm_prefill=quantize_extra("esm_prefill", pk, steps=10, haar=True))
    elif args.only == "decode_fibquant":
        r = {f"{b / 2:g}": fq_decode_extra(pk, b) for b in (2, 4, 6)}
    elif args.only == "quality_fibquant":
        r = dict(llama_decode=fq_quality_extra("llama_decode"),
                 llama_decode_without_outliers=fq_quality_extra(
                     "llama_decode", overrides=dict(n_outliers=0, sigma_scale=None)))
    else:
        from rotated_codebook_kv_tq_b200 import synth
        if args.search_rows:
            synth.VECTOR_SEARCH = synth.VECTOR_SEARCH.scaled(n=args.search_rows)
        r = search_extra(pk, steps=1)
    print(json.dumps({args.only: r}))
    return 0


def relaunch_cmd(script: str, args_list, gpus: int, port: int):
    """torchrun command that runs ``script`` on ``gpus`` ranks of one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
            script, *args_list]


def check_world(gpus: int, world: int) -> None:
    """--gpus must agree with the launcher's world size."""
    if gpus != world:
        raise SystemExit(f"bench.py: --gpus {gpus} but WORLD_SIZE={world}; launch one rank per GPU")


def main():
    args = parse_args()
    if args.only:
        return run_only(args)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # started without a launcher: start one rank per GPU ourselves
        import socket
        with socket.socket() as s:
            s.bind(("127.0.0.1", 0))
            port = s.getsockname()[1]
        return subprocess.call(relaunch_cmd(os.path.abspath(__file__), sys.argv[1:], args.gpus, port))
    world, rank, local = dist_init()
    check_world(args.gpus, world)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    import torch
    from rotated_codebook_kv_tq_b200 import synth
    from rotated_codebook_kv_tq_b200.build import build
    if rank == 0:
        build()
    barrier(world)
    torch.cuda.set_device(local)
    w = synth.WORKLOADS[args.workload]
    pk = peaks()
    K, W = args.steps, max(3, args.warmup)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    per_set = w.B * w.Hkv * ((w.T + 31) // 32 * 32) * row_bytes(w)
    n_sets = max(1, math.ceil(3 * l2 / per_set))
    bench = DecodeBench(w, n_sets)
    sampler = ClockSampler(smi_index(local))
    total, kern, per_step, clocks = time_decode(bench, K, W, world, sampler)
    total = max_over_ranks(total, world)
    kern = max_over_ranks(kern, world)
    value = weak_value(w.B * K, world, total)
    alg = bench.cache_bytes_per_step()
    achieved = alg / kern / 1e9

    K_e2e = max(10, min(K, 300))
    dt, h2d, d2h = time_e2e(bench, K_e2e, 20)
    dt = max_over_ranks(dt, world)
    e2e_value = weak_value(w.B * K_e2e, world, dt)

    line = dict(metric="compressed-KV decode tokens/s", value=value, unit="tokens/s",
                n_gpus=world, steps=K, warmup=W, ms_per_step=total / K * 1e3,
                us_per_step=total / K * 1e6, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f32", data="synthetic",
                config=dict(workload=describe(w),
                            l2=f"rotating {n_sets} compressed caches "
                               f"({n_sets * per_set / 1e6:.0f} MB > 3x L2 {l2 / 1e6:.0f} MB)",
                            parallelism=f"{world} independent replicas" if world > 1 else "1 GPU"),
                roofline=dict(bound="hbm", achieved=achieved, peak=pk["hbm"], unit="GB/s",
                              frac=achieved / pk["hbm"], traffic=ncu_traffic("dec_kernel"),
                              kernel="dec_kernel (split-K decode main loop, tcgen05)",
                              kernel_us=kern * 1e6, algorithmic_bytes=alg,
                              bytes_per_token_head=row_bytes(w),
                              peak_source=f"{pk['source']} hbm_gbs"),
                roofline_step=dict(bound="hbm", achieved=alg / (total / K) / 1e9, peak=pk["hbm"],
                                   unit="GB/s", frac=alg / (total / K) / 1e9 / pk["hbm"],
                                   note="the same algorithmic bytes over the whole step (append, "
                                        "query prologue, chunk kernel, combine)"),
                e2e=dict(value=e2e_value, unit="tokens/s", h2d_bytes_per_step=h2d,
                         d2h_bytes_per_step=d2h, us_per_step=dt / K_e2e * 1e6,
                         note="public API, pinned host buffers, host sync every step"),
                clocks=dict(sm_mhz=clocks.get("sm_mhz"), sm_max_mhz=clocks.get("sm_max_mhz"),
                            reasons=clocks.get("reasons"), samples=clocks.get("samples")),
                gpu_launches=per_step * K)

    if rank == 0 and world == 1 and not args.no_cpu:
        rows = min(w.T, 8192)
        rate, n, secs, rows = oracle_rate(bench, args.cpu_seconds, rows)
        line["cpu_baseline"] = dict(
            value=rate, unit="tokens/s", cores=blas_threads(), kind="oracle",
            sample=f"{n} oracle decode steps (quantize-append + all {w.Hq} heads) over the first "
                   f"{rows} of {w.T} tokens in {secs:.1f} s, scaled by {w.T}/{rows}")
        try:
            per = cpu_baselines()
            line["cpu_baseline"]["nproc"] = per["nproc"]
            line["cpu_baseline"]["one_thread"] = per["llama_decode"]["one_thread"]
            line["cpu_baseline"]["per_workload"] = per
        except Exception as e:  # report, do not hide
            line["cpu_baseline"]["per_workload"] = dict(error=repr(e))
    if rank == 0 and world == 1 and not args.no_extras:
        extras = {}
        try:
            extras["quantize_esm_prefill"] = quantize_extra("esm_prefill", pk)
        except Exception as e:  # report, do not hide
            extras["quantize_esm_prefill"] = dict(error=repr(e))
        try:
            extras["bidir_esm_prefill"] = bidir_extra(pk)
        except Exception as e:
            extras["bidir_esm_prefill"] = dict(error=repr(e))
        try:
            extras["decode_long_context"] = decode_extra("long_decode", pk)
        except Exception as e:
            extras["decode_long_context"] = dict(error=repr(e))
        try:
            extras["vector_search"] = search_extra(pk)
        except Exception as e:
            extras["vector_search"] = dict(error=repr(e))
        try:
            extras["decode_split_2.5bit"] = split_decode_extra(pk, "2.5")
        except Exception as e:
            extras["decode_split_2.5bit"] = dict(error=repr(e))
        try:
            extras["decode_fibquant_2bit"] = fq_decode_extra(pk, 4)
        except Exception as e:
            extras["decode_fibquant_2bit"] = dict(error=repr(e))
        line["extras"] = extras
    if rank == 0:
        print(json.dumps(line))
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
