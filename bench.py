"""Decode-step benchmark of the quantized KV cache on B200.

One step = append one new token to every sequence of a batch (quantizing a
G-token block whenever a ring fills) + decode attention for one query per
sequence over the whole cache. The workload is the Llama-3-8B-shaped GQA
layer: batch 32, 32 query / 8 KV heads, head_dim 128, context 8192, bf16
keys N(0,1) x log-normal channel magnitudes and values N(0,1), keys 2-bit per
channel in groups of 64 tokens, values 4-bit per token in groups of 64
channels, residual window 128. `--workload kv1` runs the KV1 card's BQ2_0
layout on the same shapes (2-bit keys and values per token over whole head
vectors, Hadamard rotation, 4 exact sink tokens).

Timing: W warm-up steps, then exactly K steps between barriers and device
synchronisations, timed with CUDA events on the launching stream; the job
value is the max over ranks. Each step works on the next of several
independent cache replicas, so every step streams a different cache (235 MB;
151 MB for kv1: more than the 126 MB L2) and every replica's context grows only by K/replicas
tokens. Multi-GPU runs (torchrun) give every rank its own replicas: weak
scaling, no collective on the data path.

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


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--replicas", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="llama3", choices=["llama3", "kv1"],
                    help="llama3: the headline KIVI layer (default); kv1: the same shapes with the KV1 card's BQ2_0 cache")
    ap.add_argument("--query-tokens", type=int, default=1,
                    help="query tokens per sequence and step (> 1: append them, then kvq_decode_attention_multi)")
    ap.add_argument("--page-blocks", type=int, default=0,
                    help="block records in pages of this many blocks drawn from a pool (0: contiguous)")
    return ap.parse_args()


def _bench_workload(name):
    from asymmetric_bit_kv_b200 import workloads as W

    return W.llama3_8b_gqa() if name == "llama3" else W.kv1_bq2_gqa()


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

def _oracle_worker(conn, unit, ctx, wname="llama3"):
    """One unit of the workload -- one (sequence, KV head) with its 4 query
    heads -- held in the oracle. Prefill is untimed; each 'step' command appends
    one token and runs decode attention, and replies with the tokens attended."""
    from threadpoolctl import threadpool_limits

    from asymmetric_bit_kv_b200 import workloads as W
    from oracle import kvq_oracle as O

    with threadpool_limits(1):
        wl = _bench_workload(wname)
        sinks, k_axis, rot = _layout(wl)
        g = wl.num_q_heads // wl.num_kv_heads
        unit_wl = W.Workload(wl.name, 1, g, 1, wl.head_dim, [ctx], wl.k_bits, wl.v_bits, wl.group_k, wl.group_v,
                             wl.residual, wl.kv_dtype, wl.key_dist, wl.value_std, wl.seed)
        extra = 4096
        k, v = W.generate_tokens(unit_wl, 0, [ctx + extra], seed_offset=7000 + unit)
        k = k.float().numpy()
        v = v.float().numpy()
        c = O.SequenceCache(1, wl.head_dim, wl.k_bits[0], wl.v_bits[0], wl.group_k, wl.group_v, wl.residual,
                            sinks=sinks, k_axis=k_axis, hadamard=bool(rot))
        c.append(k[:ctx], v[:ctx])
        conn.send("ready")
        i = 0
        while True:
            cmd = conn.recv()
            if cmd != "step":
                break
            q = W.generate_queries(unit_wl, 0, 1, step=i)[0].float().numpy()
            t = ctx + (i % extra)
            c.append(k[t:t + 1], v[t:t + 1])
            O.decode_attention(c, q, wl.softmax_scale)
            i += 1
            conn.send(c.length)
    conn.close()


class OracleRunner:
    """`workers` spawned processes, one workload unit each, stepped together."""

    def __init__(self, workers: int, ctx: int = 8192, wname: str = "llama3"):
        import multiprocessing as mp

        ctxm = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for u in range(workers):
            a, b = ctxm.Pipe()
            p = ctxm.Process(target=_oracle_worker, args=(b, u, ctx, wname), daemon=True)
            p.start()
            self.conns.append(a)
            self.procs.append(p)
        for c in self.conns:
            assert c.recv() == "ready"
        self.workers = workers
        self.ctx = ctx

    def step(self):
        t0 = time.perf_counter()
        for c in self.conns:
            c.send("step")
        # a unit holds one of the workload's 8 KV heads: count KV tokens
        # (all heads of a token) as unit tokens / 8
        toks = sum(c.recv() for c in self.conns) / 8
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
        return (f"{self.workers} units of the workload in parallel, one (sequence, KV head) with its 4 query heads "
                f"each (context {self.ctx}); a step = append one token + fp64 decode attention per unit; "
                f"{steps} timed steps; KV tokens counted as unit tokens / 8 KV heads")


def cpu_oracle_baseline(steps: int = 100, warmup: int = 2, wname: str = "llama3"):
    workers = max(1, min(os.cpu_count() or 1, 16))
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

def _cache_mb(wl):
    """Quantized cache bytes of one replica (MB), from the record layout of
    the method (codes + fp16 scale and zero point per group)."""
    D, G, Gv = wl.head_dim, wl.group_k, wl.group_v
    per_token_keys = _layout(wl)[1]
    kgroups = D / Gv if per_token_keys else D / G
    per_tok = wl.num_kv_heads * (D * (wl.k_bits[0] + wl.v_bits[0]) / 8 + 4 * kgroups + 4 * D / Gv)
    return wl.batch * wl.context[0] * per_tok / 1e6


def _workload_config(wl, replicas, world, mean_ctx=None):
    """The `config` object of the JSON line (shared by both arms)."""
    cfg = {
        "workload": wl.name,
        "batch": wl.batch, "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
        "head_dim": wl.head_dim, "context": wl.context[0], "k_bits": wl.k_bits[0], "v_bits": wl.v_bits[0],
        "group_k": wl.group_k, "group_v": wl.group_v, "residual": wl.residual,
        "sinks": _layout(wl)[0], "key_axis": "token" if _layout(wl)[1] else "channel", "hadamard": _layout(wl)[2],
        "kv_dtype": "bf16", "out_dtype": "bf16",
        "replicas": replicas,
        "l2": f"inputs larger than L2: each step reads a different replica's ~{_cache_mb(wl):.0f} MB cache",
        "parallelism": f"dp{world} (independent replicas per rank)",
    }
    if mean_ctx is not None:
        cfg["mean_context_timed"] = mean_ctx
    return cfg


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
    wl = _bench_workload(a.workload)
    sinks, k_axis, rot = _layout(wl)
    # tensor-core layers take the new token inside the decode launch: per-channel
    # keys without the rotation, or per-token keys over whole head vectors
    fused = (k_axis == 0 and not rot) or (k_axis == 1 and wl.group_v == wl.head_dim)
    B, Hq, Hkv, D = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    ctx = wl.context[0]
    R = a.replicas
    steps_per_rep = math.ceil((a.warmup + 2 * a.steps) / R) + 2
    cap = ctx + steps_per_rep * a.query_tokens + wl.group_k
    cfg = CacheConfig(1, B, Hq, Hkv, D, cap, wl.group_k, wl.group_v, wl.residual, wl.kv_dtype, wl.k_bits, wl.v_bits,
                      sink_tokens=sinks, k_axis=[k_axis], hadamard=rot, page_blocks=a.page_blocks,
                      pool_pages=B * -(-(cap // wl.group_k) // a.page_blocks) if a.page_blocks else 0)
    caches = []
    for r in range(R):
        c = KVCache(cfg, dev)
        k, v = W.generate_tokens(wl, 0, [ctx] * B, device=dev, seed_offset=replica_seed(rank, r))
        c.append(0, k, v, [ctx] * B)
        del k, v
        caches.append(c)
    torch.cuda.synchronize()
    gen = torch.Generator(device=dev).manual_seed(12345 + rank)
    pool = 64  # distinct per-step inputs, reused round-robin
    T = a.query_tokens  # query tokens per sequence and step (their keys and values are appended first)
    new_k = torch.randn(pool, B * T, Hkv, D, generator=gen, device=dev).to(wl.kv_dtype)
    new_v = torch.randn(pool, B * T, Hkv, D, generator=gen, device=dev).to(wl.kv_dtype)
    qs = torch.randn(pool, B * T, Hq, D, generator=gen, device=dev).to(wl.kv_dtype)
    out = torch.empty(B * T, Hq, D, dtype=wl.kv_dtype, device=dev)
    stream = torch.cuda.current_stream()
    # per-step inputs as views made once, so that the timed loop only enqueues
    views = [(new_k[j], new_v[j], qs[j]) for j in range(pool)]
    # quantized bytes per token (all KV heads): the library's block record
    # (codes, scales and zero points of G tokens of one KV head) / G
    bytes_tok = Hkv * caches[0].layout(0).record_bytes / wl.group_k

    G, Rw = wl.group_k, wl.residual

    # The device-timed loop calls the C entry point kvq_decode_step (append
    # one token per sequence + decode attention; the append rides inside the
    # decode launch unless a ring must be flushed) with arguments prepared
    # here, so that Python overhead per call stays far below the GPU time of a
    # step; the e2e leg below goes through the Python binding.
    lib = caches[0].lib
    c_step = lib.kvq_decode_step
    c_append, c_multi = lib.kvq_append, lib.kvq_decode_attention_multi
    t_lens = K.lens_array([T] * B)
    sh = stream.cuda_stream
    handles = [c.handle for c in caches]
    ptrs = [(kk.data_ptr(), vv.data_ptr(), qq.data_ptr()) for kk, vv, qq in views]
    optr, oty, scale = out.data_ptr(), 1, float(wl.softmax_scale)  # out dtype code 1 = bf16

    def step(i, r, ev=None):
        kp, vp, qp = ptrs[i % pool]
        h = handles[r]
        if ev is not None:
            ev[0].record(stream)
        if T == 1:
            st = c_step(h, 0, kp, vp, qp, optr, oty, scale, B, sh)
        else:  # the T tokens' keys and values, then the T queries of every sequence
            st = c_append(h, 0, kp, vp, t_lens, B, sh) or c_multi(h, 0, qp, optr, oty, scale, B, T, sh)
        if ev is not None:
            ev[1].record(stream)
        if st:
            raise RuntimeError(f"kvq call failed: {lib.kvq_last_error().decode()}")

    for i in range(a.warmup):
        step(i, i % R)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # Per-step accounting, computed before the timed loop so that the loop only
    # enqueues work: the (quantized, ring) lengths of every replica follow the
    # flush rule (a token that finds a full ring first moves G ring tokens into
    # the quantized cache), checked against the library's host mirror after.
    lens = [[list(caches[r].lengths(0, b)) for b in range(B)] for r in range(R)]
    plan = []  # (replica, launches, algorithmic bytes of the step, KV tokens attended)
    for i in range(a.steps):
        r = (a.warmup + i) % R
        # fused: decode + combine; a step that flushes a ring first runs the
        # quantize and ring-write kernels (unfused: ring write, split kernel,
        # combine, and the quantize kernel on a flush)
        ab, tk = T * (2 * B * Hq * D * 2 + 2 * (2 * B * Hkv * D * 2)), 0  # q in, out; new k, v in and into the ring
        ab += B * sinks * Hkv * D * 2 * 2  # the exact sink tokens
        tk += B * T * sinks
        flush = False
        for b in range(B):
            qn, n = lens[r][b]
            f = 0 if n + T <= Rw else -(-(n + T - Rw) // G)  # blocks the T appends flush
            flush = flush or f > 0
            qn, n = qn + f * G, n + T - f * G
            lens[r][b] = [qn, n]
            ab += qn * bytes_tok + n * Hkv * D * 2 * 2
            tk += T * (qn + n) - T * (T - 1) // 2  # query t sees the tokens up to its own position
        if T == 1:
            # fused: prep (plan; on a flush step also the quantize CTAs),
            # decode, combine; unfused: ring write (+ quantize on a flush),
            # split kernel, combine
            launches = 3 if fused else (3 + (1 if flush else 0))
        else:
            # append (ring write, + quantize on a flush), then decode + combine
            # per group of query tokens (at most 8 query rows per KV head)
            groups, t0, ngr = 0, 0, Hq // Hkv
            while t0 < T:
                tp = 1
                while 2 * tp * ngr <= 8 and t0 + 2 * tp <= T:
                    tp *= 2
                groups, t0 = groups + 1, t0 + tp
            launches = 1 + (1 if flush else 0) + 2 * groups
        plan.append((r, launches, ab, tk, flush))
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    launches = sum(x[1] for x in plan)
    alg_total = float(sum(x[2] for x in plan))
    tok_total = sum(x[3] for x in plan)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    e0.record(stream)
    for i in range(a.steps):
        step(a.warmup + i, plan[i][0], events[i])
    e1.record(stream)
    host_s = time.perf_counter() - h0
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    for r in range(R):
        for b in range(B):
            assert tuple(lens[r][b]) == caches[r].lengths(0, b), "step accounting out of sync with the cache"
    ms = e0.elapsed_time(e1)
    call_ms = [x[0].elapsed_time(x[1]) for x in events]
    dec_ms = sum(call_ms)
    fl = [m for m, x in zip(call_ms, plan) if x[4]]
    nf = [m for m, x in zip(call_ms, plan) if not x[4]]
    fl_us = 1e3 * sum(fl) / len(fl) if fl else 0.0
    nf_us = 1e3 * sum(nf) / len(nf) if nf else 0.0
    ms, dec_ms, fl_us, nf_us = cross_rank_max([ms, dec_ms, fl_us, nf_us], world, dev)
    value = tok_total * world / (ms / 1e3)
    achieved_gbs = alg_total / (dec_ms / 1e3) / 1e9

    # ---- end to end through the public API with host buffers ----
    # each step's k, v and q sit back to back in one pinned host buffer and
    # travel in one host-to-device copy
    e2e_steps = min(a.steps, 512)
    nk, nq = B * T * Hkv * D, B * T * Hq * D
    hkvq = torch.empty(pool, 2 * nk + nq, dtype=wl.kv_dtype).pin_memory()
    hkvq[:, :nk].copy_(new_k.reshape(pool, nk).cpu())
    hkvq[:, nk:2 * nk].copy_(new_v.reshape(pool, nk).cpu())
    hkvq[:, 2 * nk:].copy_(qs.reshape(pool, nq).cpu())
    hout = torch.empty(B * T, Hq, D, dtype=wl.kv_dtype).pin_memory()
    dkvq = torch.empty(2 * nk + nq, dtype=wl.kv_dtype, device=dev)
    dk = dkvq[:nk].view(B * T, Hkv, D)
    dv = dkvq[nk:2 * nk].view(B * T, Hkv, D)
    dq = dkvq[2 * nk:].view(B * T, Hq, D)
    tok_e2e = 0
    for i in range(e2e_steps):
        r = (a.warmup + a.steps + i) % R
        for b in range(B):
            qn, n = lens[r][b]
            f = 0 if n + T <= Rw else -(-(n + T - Rw) // G)
            qn, n = qn + f * G, n + T - f * G
            lens[r][b] = [qn, n]
            tok_e2e += T * (sinks + qn + n) - T * (T - 1) // 2
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(e2e_steps):
        r = (a.warmup + a.steps + i) % R
        j = i % pool
        dkvq.copy_(hkvq[j], non_blocking=True)
        if T == 1:
            caches[r].decode_step(0, dk, dv, dq, out, softmax_scale=wl.softmax_scale, stream=stream)
            hout.copy_(out, non_blocking=True)
        else:
            caches[r].append(0, dk, dv, [T] * B, stream=stream)
            o = caches[r].decode_attention_multi(0, dq.view(B, T, Hq, D), out_dtype=wl.kv_dtype,
                                                 softmax_scale=wl.softmax_scale, stream=stream)
            hout.copy_(o.view(B * T, Hq, D), non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1)
    e2e_ms, = cross_rank_max([e2e_ms], world, dev)
    e2e_value = tok_e2e * world / (e2e_ms / 1e3)

    result = None
    if rank == 0:
        peak, peak_kind = _peaks()
        traffic = _committed_traffic() if a.workload == "llama3" else None
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
            "dtype": "bf16",
            "dtype_detail": ("bf16 keys, values, queries and outputs; quantizer in fp32; attention on fp16 "
                             "tensor-core operands (codes exact, q*s and p*s as fp16 high and low parts) and "
                             "bf16 ones for exact tokens, fp32 accumulation and softmax"),
            "data": "synthetic (seeded; Llama-3-8B-shaped layer, no model weights)",
            "config": dict(_workload_config(wl, R, world, tok_total / (a.steps * B * T)),
                           **({"page_blocks": a.page_blocks} if a.page_blocks else {}),
                           **({"query_tokens": T} if T > 1 else {})),
            "roofline": {
                "kernel": (f"verify step: {T} tokens appended per sequence (ring write, quantize on a flush), then "
                           "decode of their queries, causal among them (split-KV decode + combine per group of query "
                           "tokens)") if T > 1 else
                          ("decode step: one token appended per sequence inside the split-KV decode kernel, + log-sum-exp "
                           "combine, per call (a step in which rings are full first runs the flush kernel that quantizes "
                           "their oldest G tokens)") if fused else
                          ("decode step: ring write, CUDA-core split-KV decode kernel and log-sum-exp combine, per call "
                           "(a ring flush adds the quantize kernel)"),
                "bound": "hbm",
                "achieved": achieved_gbs,
                "peak": peak,
                "unit": "GB/s",
                "frac": achieved_gbs / peak,
                "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                "frac_of_8tbs_nominal": achieved_gbs / 8000.0,
                "traffic": traffic,
                "decode_us_per_call": dec_ms / a.steps * 1e3,
                "flush_step_us": fl_us if fl else None,
                "flush_steps": len(fl),
                "nonflush_step_us": nf_us if nf else None,
                "nonflush_steps": len(nf),
                "host_enqueue_us_per_step": host_s / a.steps * 1e6,
                "alg_bytes_per_call": alg_total / a.steps,
            },
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": int((dk.numel() + dv.numel() + dq.numel()) * 2),
                    "d2h_bytes_per_step": int(out.numel() * 2), "steps": e2e_steps},
            "gpu_launches": launches,
            "clocks": clk,
        }
    del caches
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def _kernel_source_hash():
    import glob
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "asymmetric_bit_kv_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _committed_traffic():
    """DRAM bytes (read + write) per decode launch from the committed ncu
    capture, or None if there is none or the kernel sources changed since."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_sha256") != _kernel_source_hash():
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
    run = OracleRunner(workers, wl.context[0], wname)
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
        "data": "synthetic (seeded; Llama-3-8B-shaped layer, no model weights)",
        "config": dict(_workload_config(wl, 1, world), units_per_step=workers,
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
        cpu = cpu_oracle_baseline(wname=a.workload)   # spawned before any CUDA work in this process
    res = run_kvq(a)
    if res is not None:
        res["cpu_baseline"] = cpu
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
