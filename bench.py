"""Decode-step benchmark of the quantized KV cache on B200.

One step = append one new token to every sequence of a batch (quantizing a
G-token block whenever a ring fills) + decode attention for one query per
sequence over the whole cache, in every layer of the workload. Workloads
(`--workload`, synthetic and seeded, shapes of the models named):

* llama3 (default, the headline): Llama-3-8B-shaped GQA layer, batch 32,
  32 query / 8 KV heads, head_dim 128, context 8192, bf16 keys N(0,1) x
  log-normal channel magnitudes, values N(0,1); keys 2-bit per channel in
  groups of 64 tokens, values 4-bit per token in groups of 64 channels,
  residual window 128.
* tiny: 1 sequence, 8 heads (MHA), context 1024, fp16, K2/V2 in groups of
  32, residual 32 (the oracle's small case).
* llama2: Llama-2-7B-shaped MHA layer, batch 8, 32 heads, context 4096,
  K2/V2 in groups of 32, residual 128; 256 steps by default, each timed as
  its append and its attention separately.
* long: one sequence of 131072 tokens, 32/8 heads, K2/V2 in groups of 128,
  residual 128; plus a 4096-token prefill chunk appended to an empty
  sequence in one call, timed on its own.
* qwen3: Qwen3-8B-shaped 36 layers, 64 ragged sequences (context uniform in
  [1024, 32768]), 32/8 heads, K4/V2 (layers 0-3 K8/V4) in groups of 64,
  residual 64; paged block records; a step runs every layer.
* kv1: the llama3 shapes with the KV1 card's BQ2_0 cache (2-bit keys and
  values per token over whole head vectors, Hadamard rotation, 4 sinks).

Timing: one priming step per cache replica (after the prefill every ring is
full, so a replica's first step flushes all of its sequences; the priming
steps are timed and reported on their own), W warm-up steps, then exactly K
steps between barriers and device synchronisations, timed with CUDA events
on the launching stream; the job
value is the max over ranks. Steps cycle over independent cache replicas
whose total size exceeds the 126 MB L2 many times over, so no step finds its
cache in L2, and each replica grows by only K/replicas tokens. Multi-GPU
runs (torchrun, or `--gpus N`, which launches them) give every rank its own
replicas: weak scaling, no collective on the data path.

`--impl reference` times the CPU oracle (the plain restatement of the method
used by the tests) on the host cores instead, on a bounded sample of the same
workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention: KV tokens/s and achieved HBM GB/s vs B200 peak"
UNIT = "KV tokens/s"

# Per workload: cache replicas, default steps / warm-up, page size (0:
# contiguous records), and what else is timed.
SPECS = {
    "llama3": dict(replicas=16, steps=2048, warmup=32, page_blocks=0),
    "kv1": dict(replicas=16, steps=2048, warmup=32, page_blocks=0),
    "tiny": dict(replicas=256, steps=2048, warmup=32, page_blocks=0),
    "llama2": dict(replicas=16, steps=256, warmup=8, page_blocks=0, split_append=True),
    "long": dict(replicas=16, steps=512, warmup=8, page_blocks=0, prefill_chunk=True),
    "qwen3": dict(replicas=1, steps=16, warmup=3, page_blocks=16),
}


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: the workload's)")
    ap.add_argument("--warmup", type=int, default=None, help="warm-up steps (default: the workload's)")
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--replicas", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="llama3", choices=sorted(SPECS))
    ap.add_argument("--query-tokens", type=int, default=1,
                    help="query tokens per sequence and step (> 1: append them, then kvq_decode_attention_multi)")
    ap.add_argument("--page-blocks", type=int, default=None,
                    help="block records in pages of this many blocks drawn from a pool (0: contiguous)")
    a = ap.parse_args()
    spec = SPECS[a.workload]
    a.steps = spec["steps"] if a.steps is None else a.steps
    a.warmup = spec["warmup"] if a.warmup is None else a.warmup
    a.replicas = spec["replicas"] if a.replicas is None else a.replicas
    a.page_blocks = spec["page_blocks"] if a.page_blocks is None else a.page_blocks
    return a


def _bench_workload(name):
    from asymmetric_bit_kv_b200 import workloads as W

    return {"llama3": W.llama3_8b_gqa, "kv1": W.kv1_bq2_gqa, "tiny": W.tiny_mha, "llama2": W.llama2_7b_mha,
            "long": W.long_context_gqa, "qwen3": W.qwen3_8b_layers}[name]()


def _layout(wl):
    """(sinks, k_axis, hadamard) of a workload's cache."""
    return wl.extra.get("sinks", 0), wl.extra.get("k_axis", [0])[0], wl.extra.get("hadamard", 0)


def _dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def cross_rank_max(values, world, device):
    """Per-rank timings -> their maximum over all ranks (every rank gets it).
    Multi-GPU numbers are the slowest rank's (weak scaling: each rank times
    its own replicas)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def replica_seed(rank, r):
    """Seed offset of cache replica r on `rank`: every rank draws its own data."""
    return 1000 * rank + r


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class _Driver:
    """The few CUDA driver calls of the end-to-end leg (asynchronous copies,
    events and stream waits on raw handles), through ctypes: a microsecond or
    two each, where torch's stream and event wrappers take several."""

    def __init__(self):
        import ctypes
        c = ctypes.CDLL("libcuda.so.1")
        P, U64, SZ, U = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_uint
        self._ct = ctypes
        self._h2d, self._d2h = c.cuMemcpyHtoDAsync_v2, c.cuMemcpyDtoHAsync_v2
        self._h2d.argtypes, self._d2h.argtypes = [U64, P, SZ, P], [P, U64, SZ, P]
        self._rec, self._wait = c.cuEventRecord, c.cuStreamWaitEvent
        self._rec.argtypes, self._wait.argtypes = [P, P], [P, P, U]
        self._create, self._destroy = c.cuEventCreate, c.cuEventDestroy_v2
        self._create.argtypes, self._destroy.argtypes = [ctypes.POINTER(P), U], [P]
        for f in (self._h2d, self._d2h, self._rec, self._wait, self._create, self._destroy):
            f.restype = ctypes.c_int

    def event(self):
        e = self._ct.c_void_p()
        if self._create(self._ct.byref(e), 2):  # CU_EVENT_DISABLE_TIMING
            raise RuntimeError("cuEventCreate failed")
        return e.value

    def destroy(self, e):
        self._destroy(e)

    def htod(self, dst, src, n, s):
        return self._h2d(dst, src, n, s)

    def dtoh(self, dst, src, n, s):
        return self._d2h(dst, src, n, s)

    def record(self, e, s):
        return self._rec(e, s)

    def wait(self, s, e):
        return self._wait(s, e, 0)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            import atexit

            atexit.register(lambda pr=self.proc: pr.poll() is None and pr.terminate())
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# CPU oracle baseline (host cores, spawned worker processes)
# --------------------------------------------------------------------------

def _oracle_unit(wname):
    """(context, layer) of the oracle's unit of a workload: its (median)
    context, in a layer of its most common bit widths."""
    wl = _bench_workload(wname)
    ctx = sorted(wl.context)[len(wl.context) // 2]
    layer = 4 if wl.num_layers > 4 else 0
    return ctx, layer


def _oracle_worker(conn, unit, wname="llama3"):
    """One unit of the workload -- one (sequence, KV head) with its query
    heads -- held in the oracle. Prefill is untimed; each 'step' command appends
    one token and runs decode attention, and replies with the tokens attended."""
    from threadpoolctl import threadpool_limits

    from asymmetric_bit_kv_b200 import workloads as W
    from oracle import kvq_oracle as O

    with threadpool_limits(1):
        wl = _bench_workload(wname)
        ctx, layer = _oracle_unit(wname)
        sinks, k_axis, rot = _layout(wl)
        g = wl.num_q_heads // wl.num_kv_heads
        unit_wl = W.Workload(wl.name, 1, g, 1, wl.head_dim, [ctx], wl.k_bits, wl.v_bits, wl.group_k, wl.group_v,
                             wl.residual, wl.kv_dtype, wl.key_dist, wl.value_std, wl.seed,
                             num_layers=wl.num_layers, outliers_per_head=wl.outliers_per_head,
                             outlier_scale=wl.outlier_scale, outlier_channels=wl.outlier_channels)
        extra = 4096
        k, v = W.generate_tokens(unit_wl, layer, [ctx + extra], seed_offset=7000 + unit)
        k = k.float().numpy()
        v = v.float().numpy()
        c = O.SequenceCache(1, wl.head_dim, wl.k_bits[layer], wl.v_bits[layer], wl.group_k, wl.group_v,
                            wl.residual, sinks=sinks, k_axis=k_axis, hadamard=bool(rot))
        c.append(k[:ctx], v[:ctx])
        conn.send("ready")
        i = 0
        while True:
            cmd = conn.recv()
            if cmd != "step":
                break
            q = W.generate_queries(unit_wl, layer, 1, step=i)[0].float().numpy()
            t = ctx + (i % extra)
            c.append(k[t:t + 1], v[t:t + 1])
            O.decode_attention(c, q, wl.softmax_scale)
            i += 1
            conn.send(c.length)
    conn.close()


class OracleRunner:
    """`workers` spawned processes, one workload unit each, stepped together."""

    def __init__(self, workers: int, wname: str = "llama3"):
        import multiprocessing as mp

        ctxm = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for u in range(workers):
            a, b = ctxm.Pipe()
            p = ctxm.Process(target=_oracle_worker, args=(b, u, wname), daemon=True)
            p.start()
            self.conns.append(a)
            self.procs.append(p)
        for c in self.conns:
            assert c.recv() == "ready"
        self.workers = workers
        self.wname = wname
        self.hkv = _bench_workload(wname).num_kv_heads

    def step(self):
        t0 = time.perf_counter()
        for c in self.conns:
            c.send("step")
        # a unit holds one of the workload's KV heads: count KV tokens (all
        # heads of a token) as unit tokens / Hkv
        toks = sum(c.recv() for c in self.conns) / self.hkv
        return toks, time.perf_counter() - t0

    def close(self):
        for c in self.conns:
            try:
                c.send("stop")
            except Exception:
                pass
        for p in self.procs:
            p.join(timeout=10)

    def describe(self, steps):
        wl = _bench_workload(self.wname)
        ctx, layer = _oracle_unit(self.wname)
        g = wl.num_q_heads // wl.num_kv_heads
        return (f"{self.workers} units of the workload in parallel, one (sequence, KV head) with its {g} query "
                f"head(s) each (context {ctx}, layer {layer}'s bits); a step = append one token + fp64 decode "
                f"attention per unit; {steps} timed steps; KV tokens counted as unit tokens / {self.hkv} KV heads")


def _oracle_steps(wname):
    """Oracle steps of a bounded baseline sample (about 10-30 s of host work):
    fewer for longer contexts."""
    ctx, _ = _oracle_unit(wname)
    return max(3, min(100, int(100 * 8192 / max(ctx, 1024))))


def cpu_oracle_baseline(wname="llama3", steps=None, warmup=2):
    workers = max(1, min(os.cpu_count() or 1, 16))
    steps = _oracle_steps(wname) if steps is None else steps
    run = OracleRunner(workers, wname=wname)
    try:
        for _ in range(warmup):
            run.step()
        toks, secs = 0, 0.0
        for _ in range(steps):
            t, s = run.step()
            toks += t
            secs += s
    finally:
        run.close()
    res = {"value": toks / secs, "unit": UNIT, "cores": workers, "kind": "oracle", "sample": run.describe(steps)}
    # the same unit work on one core alone (a few steps)
    one = OracleRunner(1, wname=wname)
    try:
        one.step()
        toks1, secs1 = 0, 0.0
        for _ in range(max(3, steps // 10)):
            t, s = one.step()
            toks1 += t
            secs1 += s
    finally:
        one.close()
    res["value_1_core"] = toks1 / secs1
    return res


# --------------------------------------------------------------------------
# the library arm
# --------------------------------------------------------------------------

def _workload_config(wl, a, world, mean_ctx=None, cache_mb=None):
    """The `config` object of the JSON line (shared by both arms)."""
    ctx = wl.context
    cfg = {
        "workload": wl.name,
        "batch": wl.batch, "num_layers": wl.num_layers, "num_q_heads": wl.num_q_heads,
        "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
        "context": ctx[0] if len(set(ctx)) == 1 else {"min": min(ctx), "max": max(ctx),
                                                       "mean": sum(ctx) / len(ctx)},
        "k_bits": wl.k_bits[0] if len(set(wl.k_bits)) == 1 else wl.k_bits,
        "v_bits": wl.v_bits[0] if len(set(wl.v_bits)) == 1 else wl.v_bits,
        "group_k": wl.group_k, "group_v": wl.group_v, "residual": wl.residual,
        "sinks": _layout(wl)[0], "key_axis": "token" if _layout(wl)[1] else "channel", "hadamard": _layout(wl)[2],
        "kv_dtype": str(wl.kv_dtype).replace("torch.", ""), "out_dtype": str(wl.kv_dtype).replace("torch.", ""),
        "replicas": a.replicas,
        "parallelism": f"dp{world} (independent replicas per rank)",
    }
    if cache_mb is not None:
        cfg["l2"] = (f"inputs larger than L2: each step reads a different replica's ~{cache_mb:.0f} MB cache "
                     f"({a.replicas} replicas, {a.replicas * cache_mb:.0f} MB in all)")
    if a.page_blocks:
        cfg["page_blocks"] = a.page_blocks
    if a.query_tokens > 1:
        cfg["query_tokens"] = a.query_tokens
    if mean_ctx is not None:
        cfg["mean_context_timed"] = mean_ctx
    return cfg


def _flushes(n, T, R, G):
    """Blocks a ring of n tokens (R slots) flushes when T tokens arrive one by one."""
    return 0 if n + T <= R else -(-(n + T - R) // G)


def run_kvq(a):
    import torch
    import torch.distributed as dist

    from asymmetric_bit_kv_b200 import CacheConfig, KVCache
    from asymmetric_bit_kv_b200 import kvq as K
    from asymmetric_bit_kv_b200 import workloads as W

    rank, world, local = _dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # clocks are sampled from here on (cache fill, priming, warm-up and the
    # timed steps): nvidia-smi takes a while to start, and no idle pause
    # precedes the timed loop
    clocks = ClockSampler(local)
    clocks.start()
    spec = SPECS[a.workload]
    wl = _bench_workload(a.workload)
    sinks, k_axis, rot = _layout(wl)
    B, Hq, Hkv, D, NL = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.num_layers
    G, Rw = wl.group_k, wl.residual
    ctx = list(wl.context)
    R = a.replicas
    T = a.query_tokens  # query tokens per sequence and step (their keys and values are appended first)
    split_append = spec.get("split_append", False) and T == 1
    # steps per replica: priming, warm-up, the timed loop, the per-step pass
    # (up to 256 steps) and the e2e leg (up to 512 steps)
    steps_per_rep = math.ceil((a.warmup + a.steps + min(a.steps, 256) + min(a.steps, 512)) / R) + 3
    cap = max(ctx) + sinks + steps_per_rep * T + G
    pool_pages = 0
    if a.page_blocks:
        pool_pages = sum(-(-((c + steps_per_rep * T + G) // G + 1) // a.page_blocks) for c in ctx) + B
    cfg = CacheConfig(NL, B, Hq, Hkv, D, cap, G, wl.group_v, Rw, wl.kv_dtype, wl.k_bits, wl.v_bits,
                      sink_tokens=sinks, k_axis=[k_axis] * NL, hadamard=rot, page_blocks=a.page_blocks,
                      pool_pages=pool_pages)
    caches = []
    for r in range(R):
        c = KVCache(cfg, dev)
        for layer in range(NL):
            k, v = W.generate_tokens(wl, layer, ctx, device=dev, seed_offset=replica_seed(rank, r))
            c.append(layer, k, v, ctx)
            del k, v
        caches.append(c)
    torch.cuda.synchronize()
    lib = caches[0].lib
    gen = torch.Generator(device=dev).manual_seed(12345 + rank)
    pool = 64  # distinct per-step inputs, reused round-robin
    new_k = torch.randn(pool, B * T, Hkv, D, generator=gen, device=dev).to(wl.kv_dtype)
    new_v = torch.randn(pool, B * T, Hkv, D, generator=gen, device=dev).to(wl.kv_dtype)
    qs = torch.randn(pool, B * T, Hq, D, generator=gen, device=dev).to(wl.kv_dtype)
    out = torch.empty(B * T, Hq, D, dtype=wl.kv_dtype, device=dev)
    stream = torch.cuda.current_stream()
    oty = K.KVQ_BF16 if wl.kv_dtype == torch.bfloat16 else K.KVQ_F16
    scale = float(wl.softmax_scale)
    # quantized bytes per token (all KV heads) of each layer: the library's
    # block record (codes, scales and zero points of G tokens of one KV head) / G
    bytes_tok = [Hkv * caches[0].layout(layer).record_bytes / G for layer in range(NL)]
    # layers on a tensor-core kernel take the new token inside the decode
    # launch (kvq_decode_step); the library says which kernel a layer runs
    kernels = [caches[0].decode_kernel(layer) for layer in range(NL)]
    fused = all(kn != "cuda_core" for kn in kernels)

    # The device-timed loop calls the C entry points with arguments prepared
    # here, so that Python overhead per call stays far below the GPU time of a
    # step; the e2e leg below goes through the Python binding.
    c_step, c_append, c_decode, c_multi = (lib.kvq_decode_step, lib.kvq_append, lib.kvq_decode_attention,
                                           lib.kvq_decode_attention_multi)
    t_lens = K.lens_array([T] * B)
    sh = stream.cuda_stream
    handles = [c.handle for c in caches]
    ptrs = [(kk.data_ptr(), vv.data_ptr(), qq.data_ptr()) for kk, vv, qq in zip(new_k, new_v, qs)]
    optr = out.data_ptr()

    lib_s = [0.0]  # host time inside the library's entry points (ctypes calls included)

    def timed(fn, *args):
        t = time.perf_counter()
        st = fn(*args)
        lib_s[0] += time.perf_counter() - t
        return st

    def step(i, r, ev=None):
        """One step on replica r: every layer; ev = (start, after append, end)
        events (the middle one only with split_append)."""
        kp, vp, qp = ptrs[i % pool]
        h = handles[r]
        if ev is not None:
            ev[0].record(stream)
        st = 0
        for layer in range(NL):
            if split_append:
                st = st or timed(c_append, h, layer, kp, vp, t_lens, B, sh)
                if ev is not None and layer == NL - 1:
                    ev[1].record(stream)
                st = st or timed(c_decode, h, layer, qp, optr, oty, scale, B, sh)
            elif T == 1:
                st = st or timed(c_step, h, layer, kp, vp, qp, optr, oty, scale, B, sh)
            else:  # the T tokens' keys and values, then the T queries of every sequence
                st = st or timed(c_append, h, layer, kp, vp, t_lens, B, sh) or \
                    timed(c_multi, h, layer, qp, optr, oty, scale, B, T, sh)
        if ev is not None:
            ev[2].record(stream)
        if st:
            raise RuntimeError(f"kvq call failed: {lib.kvq_last_error().decode()}")

    # Priming: one step on every replica before the warm-up steps. After the
    # prefill every sequence's ring is full (the context is a multiple of G),
    # so the first step on a replica flushes every sequence; in steady state a
    # sequence flushes once every G / T steps. Without priming a short run
    # (fewer steps than replicas) would time almost only first-visit flushes.
    # The priming steps are timed on their own and reported.
    mirror0 = [[caches[r].lengths(layer, 0)[0] for layer in range(NL)] for r in range(R)]
    prime_ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(R)]
    for r in range(R):
        step(r, r, prime_ev[r])
    torch.cuda.synchronize()
    prime_flush = [any(caches[r].lengths(layer, 0)[0] > mirror0[r][layer] for layer in range(NL)) for r in range(R)]
    prime_ms = [e[0].elapsed_time(e[2]) for e in prime_ev]
    for i in range(a.warmup):
        step(R + i, i % R)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # Per-step accounting, computed before the timed loop so that the loop only
    # enqueues work: the (quantized, ring) state of every replica follows
    # the flush rule (a token that finds a full ring first moves G ring tokens
    # into the quantized cache), checked against the library's host mirror after.
    lens = [[[list(caches[r].lengths(layer, b)) for b in range(B)] for layer in range(NL)] for r in range(R)]

    def make_plan(first, nsteps):
        """(replica, algorithmic bytes, KV tokens attended, any flush) of
        steps first .. first + nsteps - 1, advancing lens."""
        plan = []
        for i in range(first, first + nsteps):
            r = i % R
            ab = tk = 0
            flush = False
            for layer in range(NL):
                ab += T * (2 * B * Hq * D * 2 + 2 * (2 * B * Hkv * D * 2))  # q in, out; new k, v in and into the ring
                ab += B * sinks * Hkv * D * 2 * 2  # the exact sink tokens
                tk += B * T * sinks
                lflush = False
                for b in range(B):
                    qn, n = lens[r][layer][b]
                    f = _flushes(n, T, Rw, G)
                    lflush = lflush or f > 0
                    qn, n = qn + f * G, n + T - f * G
                    lens[r][layer][b] = [qn, n]
                    ab += qn * bytes_tok[layer] + n * Hkv * D * 2 * 2
                    tk += T * (qn + n) - T * (T - 1) // 2  # query t sees the tokens up to its own position
                flush = flush or lflush
            plan.append((r, ab, tk, flush))
        return plan

    def check_mirror():
        for r in range(R):
            for layer in range(NL):
                for b in range(B):
                    assert tuple(lens[r][layer][b]) == caches[r].lengths(layer, b), "step accounting out of sync"

    plan = make_plan(a.warmup, a.steps)
    alg_total = float(sum(x[1] for x in plan))
    tok_total = sum(x[2] for x in plan)

    # The timed loop: exactly K steps between one pair of events (no event
    # inside, so that nothing but the steps runs on the stream).
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # kernels the timed steps enqueue, as the library counts them
    launches0 = sum(c.kernel_launches() for c in caches)
    h0 = time.perf_counter()
    e0.record(stream)
    # host cost of enqueueing a step: the first nburst steps, about 64 library
    # calls (later ones also wait for room in the launch queue once the GPU
    # falls behind)
    nburst = max(1, min(a.steps, 32, 64 // NL))
    burst_s = burst_lib_s = 0.0
    lib_s[0] = 0.0
    for i in range(a.steps):
        step(a.warmup + i, plan[i][0])
        if i + 1 == nburst:
            burst_s = time.perf_counter() - h0
            burst_lib_s = lib_s[0]
    e1.record(stream)
    host_s = time.perf_counter() - h0
    launches = sum(c.kernel_launches() for c in caches) - launches0
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    check_mirror()
    ms = e0.elapsed_time(e1)

    # A second pass of up to 256 steps, each between its own events: how the
    # step time splits into flush and non-flush steps (and append and
    # attention with split_append). Not part of `value`.
    n2 = min(a.steps, 256)
    plan2 = make_plan(a.warmup + a.steps, n2)
    events = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(n2)]
    for i in range(n2):
        step(a.warmup + a.steps + i, plan2[i][0], events[i])
    torch.cuda.synchronize()
    check_mirror()
    call_ms = [x[0].elapsed_time(x[2]) for x in events]
    app_ms = [x[0].elapsed_time(x[1]) for x in events] if split_append else [0.0]
    fl = [m for m, x in zip(call_ms, plan2) if x[3]]
    nf = [m for m, x in zip(call_ms, plan2) if not x[3]]
    call_us = 1e3 * sum(call_ms) / len(call_ms)
    fl_us = 1e3 * sum(fl) / len(fl) if fl else 0.0
    nf_us = 1e3 * sum(nf) / len(nf) if nf else 0.0
    app_us = 1e3 * sum(app_ms) / len(app_ms)
    ms, call_us, fl_us, nf_us, app_us = cross_rank_max([ms, call_us, fl_us, nf_us, app_us], world, dev)
    value = tok_total * world / (ms / 1e3)
    achieved_gbs = alg_total / (ms / 1e3) / 1e9

    # ---- a prefill chunk: one kvq_append of 4096 tokens to an empty sequence
    prefill = None
    if spec.get("prefill_chunk"):
        chunk = wl.extra.get("prefill_chunk", 4096)
        pc = CacheConfig(1, 1, Hq, Hkv, D, chunk + G, G, wl.group_v, Rw, wl.kv_dtype, wl.k_bits[:1], wl.v_bits[:1],
                         sink_tokens=sinks, k_axis=[k_axis], hadamard=rot)
        pcs = [KVCache(pc, dev) for _ in range(8)]
        ck, cv = W.generate_tokens(wl, 0, [chunk], device=dev, seed_offset=99)
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2, written before each run
        pt = []
        for rep in range(8 + 3):
            c = pcs[rep % 8]
            c.reset()
            flush_buf.fill_(rep & 0xff)
            pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            pa.record(stream)
            c.append(0, ck, cv, [chunk])
            pb.record(stream)
            pt.append((pa, pb))
        torch.cuda.synchronize()
        us = sorted(x.elapsed_time(y) * 1e3 for x, y in pt[3:])
        qb = pcs[0].lengths(0, 0)[0] // G
        in_b = chunk * Hkv * D * 2 * 2
        out_b = qb * G * bytes_tok[0] + (chunk - qb * G) * Hkv * D * 2 * 2
        prefill = {"tokens": chunk, "us_median": us[len(us) // 2], "bytes_in": in_b, "bytes_out": int(out_b),
                   "achieved_gbs": (in_b + out_b) / (us[len(us) // 2] * 1e-6) / 1e9,
                   "what": "one kvq_append of the chunk to an empty sequence (quantize kernel + ring write), "
                           "L2 flushed before each run"}
        del pcs, flush_buf, ck, cv

    # ---- end to end through the public API with host buffers ----
    # each step's k, v and q sit back to back in one pinned host buffer and
    # travel in one host-to-device copy; the last layer's output comes back.
    # The copies run on their own stream, double-buffered, so that step i+1's
    # inputs go up and step i's output comes down while the GPU computes
    # (events order every reuse of a buffer); all of them lie inside the
    # timed region.
    e2e_steps = min(a.steps, 512)
    e2e_warm = 3  # untimed steps through the same path first (first-call costs of the binding and driver calls)
    nk, nq = B * T * Hkv * D, B * T * Hq * D
    hkvq = torch.empty(pool, 2 * nk + nq, dtype=wl.kv_dtype).pin_memory()
    hkvq[:, :nk].copy_(new_k.reshape(pool, nk).cpu())
    hkvq[:, nk:2 * nk].copy_(new_v.reshape(pool, nk).cpu())
    hkvq[:, 2 * nk:].copy_(qs.reshape(pool, nq).cpu())
    hout = torch.empty(2, B * T, Hq, D, dtype=wl.kv_dtype).pin_memory()
    dkvq = [torch.empty(2 * nk + nq, dtype=wl.kv_dtype, device=dev) for _ in range(2)]
    douts = [torch.empty(B * T, Hq, D, dtype=wl.kv_dtype, device=dev) for _ in range(2)]
    e2e_first = a.warmup + a.steps + n2  # step index of the first e2e step (warm-up included)
    tok_e2e = 0
    for i in range(e2e_warm + e2e_steps):
        r = (e2e_first + i) % R
        for layer in range(NL):
            for b in range(B):
                qn, n = lens[r][layer][b]
                f = _flushes(n, T, Rw, G)
                qn, n = qn + f * G, n + T - f * G
                lens[r][layer][b] = [qn, n]
                if i >= e2e_warm:
                    tok_e2e += T * (sinks + qn + n) - T * (T - 1) // 2
    cstream = torch.cuda.Stream(device=dev)
    drv = _Driver()
    cs, ms_ = cstream.cuda_stream, stream.cuda_stream
    ev_in = [drv.event() for _ in range(2)]    # inputs of the buffer landed
    ev_used = [drv.event() for _ in range(2)]  # the step that read / wrote the buffer is done
    ev_out = [drv.event() for _ in range(2)]   # its output copied to the host
    ev_start = drv.event()
    in_bytes = (2 * nk + nq) * 2
    out_bytes = B * T * Hq * D * 2
    # k, v and q views of each input buffer, made once
    views = [(x[:nk].view(B * T, Hkv, D), x[nk:2 * nk].view(B * T, Hkv, D), x[2 * nk:].view(B * T, Hq, D),
              x[2 * nk:].view(B, T, Hq, D)) for x in dkvq]

    def e2e_run(first, n):
        """Steps first .. first + n - 1 of the e2e sequence, copies included;
        returns the OR of the driver calls' status codes."""
        rc = drv.record(ev_start, ms_) | drv.wait(cs, ev_start)

        def upload(i):
            j = i % 2
            r_ = drv.wait(cs, ev_used[j]) if i >= 2 else 0
            return r_ | drv.htod(dkvq[j].data_ptr(), hkvq[(first + i) % pool].data_ptr(), in_bytes, cs) | drv.record(
                ev_in[j], cs)

        rc |= upload(0)
        for i in range(n):
            j = i % 2
            r = (e2e_first + first + i) % R
            if i + 1 < n:
                rc |= upload(i + 1)
            rc |= drv.wait(ms_, ev_in[j])
            if i >= 2:
                rc |= drv.wait(ms_, ev_out[j])  # step i - 2's output has left douts[j]
            dk, dv, dq, dq_t = views[j]
            o = douts[j]
            for layer in range(NL):
                if T == 1:
                    caches[r].decode_step(layer, dk, dv, dq, o, softmax_scale=wl.softmax_scale, stream=stream)
                else:
                    caches[r].append(layer, dk, dv, [T] * B, stream=stream)
                    o = caches[r].decode_attention_multi(layer, dq_t, out_dtype=wl.kv_dtype,
                                                         softmax_scale=wl.softmax_scale, stream=stream)
                    o.record_stream(cstream)  # allocated per call on `stream`, read by the copy stream
            rc |= drv.record(ev_used[j], ms_) | drv.wait(cs, ev_used[j])
            rc |= drv.dtoh(hout[j].data_ptr(), o.data_ptr(), out_bytes, cs) | drv.record(ev_out[j], cs)
        stream.wait_stream(cstream)
        return rc

    rc = e2e_run(0, e2e_warm)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    rc |= e2e_run(e2e_warm, e2e_steps)
    f1.record(stream)
    torch.cuda.synchronize()
    if rc:
        raise RuntimeError("a CUDA driver call of the end-to-end leg failed")
    for e in ev_in + ev_used + ev_out + [ev_start]:
        drv.destroy(e)
    e2e_ms, = cross_rank_max([f0.elapsed_time(f1)], world, dev)
    e2e_value = tok_e2e * world / (e2e_ms / 1e3)

    result = None
    if rank == 0:
        peak, peak_kind = _peaks()
        cache_mb = sum(c * bytes_tok[layer] for layer in range(NL) for c in ctx) / 1e6
        if T > 1:
            kernel = (f"verify step: {T} tokens appended per sequence (ring write, quantize on a flush), then decode "
                      "of their queries, causal among them (split-KV decode + combine per group of query tokens)")
        elif split_append:
            kernel = ("append (ring write; the quantize kernel when a ring fills), then the split-KV decode kernel "
                      "and the log-sum-exp combine")
        elif fused:
            kernel = ("decode step: one token appended per sequence inside the tensor-core split-KV decode kernel, "
                      "+ log-sum-exp combine (a step in which rings are full first runs the flush kernel that "
                      "quantizes their oldest G tokens)")
        else:
            kernel = ("decode step: ring write (+ quantize when a ring fills), CUDA-core split-KV decode kernel and "
                      "log-sum-exp combine")
        result = {
            "metric": METRIC,
            "value": value,
            "unit": UNIT,
            "n_gpus": world,
            "steps": a.steps,
            "warmup": a.warmup,
            "ms_per_step": ms / a.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": str(wl.kv_dtype).replace("torch.", ""),
            "dtype_detail": (f"{str(wl.kv_dtype).replace('torch.', '')} keys, values, queries and outputs; quantizer "
                             "in fp32; attention on fp16 tensor-core operands (codes exact, q*s and p*s as fp16 high "
                             "and low parts) or fp32 CUDA-core arithmetic, fp32 accumulation and softmax"),
            "data": f"synthetic (seeded; {wl.name}, model-shaped, no model weights)",
            "config": _workload_config(wl, a, world, tok_total / (a.steps * NL * B * T), cache_mb),
            "roofline": {
                "kernel": kernel,
                "bound": "hbm",
                "achieved": achieved_gbs,
                "peak": peak,
                "unit": "GB/s",
                "frac": achieved_gbs / peak,
                "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                "frac_of_8tbs_nominal": achieved_gbs / 8000.0,
                "traffic": _committed_traffic(a.workload),
                "timing": ("achieved = algorithmic bytes of the K timed steps / their device time (one event "
                           "pair around the loop); step_call_us and the flush split come from a separate pass of "
                           "up to 256 steps, each between its own events"),
                "step_us": ms / a.steps * 1e3,
                "step_call_us": call_us,
                "flush_step_us": fl_us if fl else None,
                "flush_steps": len(fl),
                "nonflush_step_us": nf_us if nf else None,
                "nonflush_steps": len(nf),
                "host_enqueue_us_per_step": burst_lib_s / nburst * 1e6,
                "host_step_us_per_step": burst_s / nburst * 1e6,
                "host_loop_us_per_step": host_s / a.steps * 1e6,
                "prime_step_us": 1e3 * statistics.median(prime_ms),
                "prime_steps_flushing": sum(prime_flush),
                "alg_bytes_per_step": alg_total / a.steps,
            },
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": int(in_bytes), "d2h_bytes_per_step": int(out_bytes),
                    "steps": e2e_steps, "warmup_steps": e2e_warm,
                    "copies": "one pinned host-to-device and one device-to-host copy per step, on a copy stream "
                              "overlapped with the previous and next steps"},
            "gpu_launches": launches * world,  # every rank runs the same steps: the whole job's kernels
            "clocks": clk,
        }
        if split_append:
            result["roofline"]["append_us_per_step"] = app_us
            result["roofline"]["attention_us_per_step"] = call_us - app_us
        if prefill is not None:
            result["prefill_chunk"] = prefill
    del caches
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# Sources a decode launch's DRAM traffic depends on: the decode kernels, the
# record layout, the plan and launch code; not the quantize kernels
# (kvq_append.*) nor the static-scratch entry point (kvq_noalloc.cu).
_NOT_DECODE = ("kvq_append.cu", "kvq_append.cuh", "kvq_noalloc.cu")


def _kernel_source_hash():
    import glob
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "asymmetric_bit_kv_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        if os.path.basename(f) in _NOT_DECODE:
            continue
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _committed_traffic(workload="llama3"):
    """DRAM bytes (read + write) per decode launch of a workload from the
    committed ncu capture, or None if there is none or the kernel sources
    changed since."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except Exception:
        return None
    rec = rec.get(workload)
    if not rec or rec.get("source_sha256") != _kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


def run_reference(a):
    """The CPU oracle on the host cores, K steps after W warm-up steps; every
    step is a bounded sample of the workload (one unit per host core)."""
    rank, world, _ = _dist_env()
    if rank != 0:
        return None
    wname = getattr(a, "workload", "llama3")
    wl = _bench_workload(wname)
    workers = max(1, min(os.cpu_count() or 1, 16))
    t_start = time.perf_counter()
    run = OracleRunner(workers, wname)
    try:
        for _ in range(a.warmup):
            run.step()
        toks, secs = 0, 0.0
        for _ in range(a.steps):
            t, s = run.step()
            toks += t
            secs += s
    finally:
        run.close()
    value = toks / secs
    base = {"value": value, "unit": UNIT, "cores": workers, "kind": "oracle", "sample": run.describe(a.steps)}
    cfg_args = type("A", (), {"replicas": 1, "page_blocks": 0, "query_tokens": 1})()
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": 1e3 * secs / a.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": f"synthetic (seeded; {wl.name}, model-shaped, no model weights)",
        "config": dict(_workload_config(wl, cfg_args, world), units_per_step=workers,
                       l2="host run: one bounded sample of the workload per step"),
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t_start,
    }


def _launch_ranks(n):
    """Re-run this command as n ranks, one process per GPU, under
    torch.distributed.run on this node (the way a multi-GPU run is launched);
    returns its exit status."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    a = _args()
    if "WORLD_SIZE" not in os.environ and a.gpus > 1:
        sys.exit(_launch_ranks(a.gpus))
    if int(os.environ.get("WORLD_SIZE", "1")) != a.gpus:
        sys.exit(f"bench.py: --gpus {a.gpus} but WORLD_SIZE is {os.environ.get('WORLD_SIZE')}: "
                 "launch one rank per GPU (torchrun --nproc-per-node N) or let bench.py launch them")
    if a.impl == "reference":
        res = run_reference(a)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, _ = _dist_env()
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline and a.query_tokens == 1:
        cpu = cpu_oracle_baseline(a.workload)   # spawned before any CUDA work in this process
    res = run_kvq(a)
    if res is not None:
        res["cpu_baseline"] = cpu
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
