"""Benchmark of the decode-time QSA hot path on B200.

One step = compress-append of the new token(s) + indexer top-k over every
micro-block + sparse split-KV decode over the selected tokens + LSE merge,
for one batch of the named workload (default: batch 128 x 262,144-token
contexts, GQA 16/2, D 128, bf16, 2 KV splits).  The caches (K/V, compressed
keys) are built untimed and stay resident; the compressed-key scan alone
(2 GiB per step) is far larger than L2, so no flush is needed between steps.

Prints ONE JSON line on rank 0.  ``--impl reference`` times the CPU oracle
(the reference arm of this method: there is no runnable reference code) on
a bounded sample of the same workload.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QSA decode queries/s and achieved HBM GB/s (% of B200 peak) at 256k ctx"
UNIT = "queries/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="b128_256k")
    ap.add_argument("--splits", type=int, default=2)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (profiling runs only)")
    ap.add_argument("--ctx", default=None,
                    help="override the workload's context lengths, e.g. fixed:16384 "
                         "(profiling runs only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--dcp", action="store_true",
                    help="decode context parallelism: the ranks share one batch, rank k attends "
                         "split k of N and the partials are all-gathered (strong scaling); "
                         "default: independent replicas (weak scaling)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the steps as eager launches instead of one CUDA graph replay")
    ap.add_argument("--cpu-queries", type=int, default=300,
                    help="oracle queries timed for the CPU baseline")
    ap.add_argument("--prefill", action="store_true",
                    help="time the sparse prefill (qsa_sparse_prefill) instead of the decode step")
    ap.add_argument("--prefill-batch", type=int, default=4)
    ap.add_argument("--prefill-ctx", type=int, default=32768)
    ap.add_argument("--prefill-chunk", type=int, default=1024,
                    help="query tokens per request: the newest tokens of each context")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# Multi-rank helpers (one process per GPU; replicas of the workload)
# ---------------------------------------------------------------------------

def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (independent replicas, weak scaling)."""
    return base_seed + rank


def max_over_ranks(value_ms: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank calls this, in the same order)."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(per_rank_units: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: units of all ranks over the slowest rank's time."""
    return world * per_rank_units * steps / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# Algorithmic bytes (what the method must move), per query and per launch
# ---------------------------------------------------------------------------

def algorithmic_bytes(w, L: int, num_splits: int) -> dict:
    """Bytes one query (one request, T query tokens) must move.

    index_topk : every competing compressed key (packed: d low bytes and d/4
                 bytes of 2-bit high fields per block), the
                 block-table entries of those pages, the indexer query and
                 the selection row written.
    sparse_decode : K and V rows of the selected tokens for every kv head,
                 the query, the block-table entries of the selected pages
                 (counted once per page of the table row already), the
                 partial outputs written.
    lse_merge  : partial outputs read, merged output written.
    """
    n = (L - w.T) // 4 + 1
    P = w.page_size
    kv_elem = {"f32": 4, "bf16": 2, "e4m3": 1}[w.kv_dtype]
    q_elem = {"f32": 4, "bf16": 2}[w.q_dtype]
    pages = math.ceil(n * 4 / P)
    topk = min(w.topk, n)
    tokens = topk * 4 + (w.T - 1)
    kc_block = w.d_idx + w.d_idx // 4
    idx = n * kc_block + pages * 4 + w.d_idx + w.topk * 4
    dec = (2 * tokens * w.Hkv * w.D * kv_elem + w.T * w.Hq * w.D * q_elem + w.topk * 4
           + num_splits * w.T * w.Hq * (w.D + 1) * 4)
    if w.kv_dtype == "e4m3":
        dec += 2 * min(tokens, math.ceil(L / P)) * w.Hkv * 4
    merge = num_splits * w.T * w.Hq * (w.D + 1) * 4 + w.T * w.Hq * (w.D + 1) * 4
    append = w.T * w.d_idx * 3 + 2 * kc_block
    return dict(index_topk=idx, sparse_decode=dec, lse_merge=merge, compress_append=append,
                total=idx + dec + merge + append)


L2_BYTES = 126 * 1000 * 1000  # B200 L2


def mean_context(w) -> float:
    """Mean context length of the workload's length distribution."""
    kind, *a = w.ctx.split(":")
    if kind == "fixed":
        return float(a[0])
    lo, hi = float(a[0]), float(a[1])
    if kind == "uniform":
        return (lo + hi) / 2
    return (hi - lo) / math.log(hi / lo)  # loguniform


def step_bytes(w, num_splits: int) -> int:
    """Algorithmic bytes of one step of the whole batch at the mean length."""
    return int(w.batch * algorithmic_bytes(w, int(mean_context(w)), num_splits)["total"])


def workload_config(w, num_splits: int, world: int, dcp: bool = False) -> dict:
    """The `config` object of the JSON line (both arms)."""
    kind, *a = w.ctx.split(":")
    sb = step_bytes(w, num_splits)
    l2 = (f"inputs larger than L2: ~{sb / 1e9:.2f} GB read per step (mostly packed "
          f"compressed keys), no flush" if sb > L2_BYTES else
          f"inputs smaller than L2 (~{sb / 1e6:.0f} MB per step), no flush: steps may hit L2")
    par = "single GPU"
    if world > 1:
        par = f"decode context parallel x{world} (NCCL all-gather)" if dcp else f"replicas x{world}"
    return {"workload": w.name, "description": w.description,
            "global_batch": w.batch * (1 if dcp else world),
            "seq_len": int(a[-1]), "query_tokens": w.T, "kv_splits": num_splits,
            "topk_blocks": w.topk, "page_size": w.page_size,
            "parallelism": par,
            "l2": l2,
            "timing": "value: K back-to-back steps (one CUDA graph of the K steps, replayed "
                      "once after an untimed replay; --no-graph: eager launches); kernel_ms and "
                      "roofline: a second, eager K-step pass with events between the kernels"}


def index_topk_traffic(batch: int):
    """DRAM bytes of one qsa_index_topk launch from the committed ncu capture
    (profiles/roofline_traffic.json), scaled by requests; None when the
    kernel source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f)
    with open(os.path.join(ROOT, t["source"]), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if not sha.startswith(t["source_sha256_prefix"]):
        return None
    return int(t["dram_bytes_per_request"]) * batch


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

REASON_KEYS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.t0 = self.t1 = self.t2 = None

    def start(self):
        q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={q}", "--format=csv,noheader",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, which: str):
        setattr(self, which, time.time())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                sm = float(parts[1].split()[0])
                smax = float(parts[2].split()[0])
            except (ValueError, IndexError):
                continue
            flags = {k: parts[5 + i].strip() == "Active" for i, k in enumerate(REASON_KEYS)}
            rows.append((ts, sm, smax, flags))
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        end = self.t2 if self.t2 is not None else self.t1
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.06 <= r[0] <= end + 0.06]
        use = inside if inside else rows
        reasons = sorted({k for r in use for k, v in r[3].items() if v})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use),
                "window": "timed region" if inside else "whole run"}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_request_inputs(w, L: int, seed: int):
    """Logical inputs of one request on the host (same recipe as the device
    generator, drawn on the CPU)."""
    from workloads.qsa_inputs import make_batch
    import numpy as np
    from oracle import qsa_ref as ref
    b = make_batch(w, "cpu", seed=seed, ctx_lens=[L])
    k_idx = b.k_idx.numpy()
    if b.k_cache.dtype.itemsize == 2:
        kst = b.k_cache.view(__import__("torch").int16).numpy().view(np.uint16)
        vst = b.v_cache.view(__import__("torch").int16).numpy().view(np.uint16)
        kind = "bf16"
    elif b.k_cache.dtype.itemsize == 1:
        kst = b.k_cache.view(__import__("torch").uint8).numpy()
        vst = b.v_cache.view(__import__("torch").uint8).numpy()
        kind = "e4m3"
    else:
        kst, vst, kind = b.k_cache.numpy(), b.v_cache.numpy(), "f32"
    table = b.block_table_host[0].numpy()
    K = ref.StoredRows(ref.depage(kst, table, L, w.page_size), kind,
                       None if b.k_scale is None else b.k_scale.numpy()[table[np.arange(L) // w.page_size]])
    V = ref.StoredRows(ref.depage(vst, table, L, w.page_size), kind,
                       None if b.v_scale is None else b.v_scale.numpy()[table[np.arange(L) // w.page_size]])
    qb = b.q[0]
    if qb.dtype.itemsize == 2:
        q = ref.bf16_bits_to_f64(qb.view(__import__("torch").int16).numpy().view(np.uint16))
    else:
        q = qb.double().numpy()
    kc = ref.compress_keys(k_idx[: L - w.T])       # cache state before the step (untimed)
    return dict(k_idx=k_idx, q_idx=b.q_idx[0].numpy(), q=q, K=K, V=V, kc_prefix=kc, L=L)


def oracle_step(w, inp: dict, num_splits: int):
    """One decode step of the oracle for one request, in the order of the GPU
    step: compress the blocks the new tokens touch, score, select, attend
    per split, merge."""
    import numpy as np
    from oracle import qsa_ref as ref
    L, T = inp["L"], w.T
    p0 = L - T
    b0 = p0 // 4
    touched = ref.compress_keys(inp["k_idx"][4 * b0: L])
    kc = np.concatenate([inp["kc_prefix"][:b0], touched])
    n_sel = ref.selection_width(L, T)
    scores = ref.block_scores(inp["q_idx"], kc, n_sel)
    sel = ref.select_blocks(scores, w.topk)
    D = w.D
    outs = []
    for t in range(T):
        toks = ref.token_set(sel, L, T, t)
        op, lp = ref.split_attention(inp["q"][t], inp["K"], inp["V"], toks, 1.0 / math.sqrt(D), L,
                                     w.page_size, num_splits)
        outs.append(ref.lse_merge(op, lp))
    return sel, outs


_ORACLE_POOL: dict = {}


def oracle_pool(w, n_distinct: int, seed: int) -> list:
    """A few requests of workload w drawn on the host (cached; untimed)."""
    from workloads.qsa_inputs import draw_ctx_lens
    import torch
    key = (w.name, n_distinct, seed)
    if key not in _ORACLE_POOL:
        lens = draw_ctx_lens(w, torch.Generator().manual_seed(seed)).tolist()
        _ORACLE_POOL[key] = [oracle_request_inputs(w, int(lens[i % len(lens)]), seed + i)
                             for i in range(n_distinct)]
    return _ORACLE_POOL[key]


def time_oracle(w, num_splits: int, n_queries: int, seed: int = 1000, n_distinct: int = 2) -> dict:
    """Times the oracle (as it stands) on n_queries decode steps of workload
    w, cycling over n_distinct host-drawn requests, on one host core; input
    generation is not timed."""
    from threadpoolctl import threadpool_limits
    import torch
    pool = oracle_pool(w, n_distinct, seed)
    elapsed = 0.0
    queries = 0
    with threadpool_limits(limits=1):
        nt = torch.get_num_threads()
        torch.set_num_threads(1)
        for i in range(n_queries):
            inp = pool[i % len(pool)]
            t0 = time.perf_counter()
            oracle_step(w, inp, num_splits)
            elapsed += time.perf_counter() - t0
            queries += w.T
        torch.set_num_threads(nt)
    return dict(value=queries / elapsed, queries=queries, seconds=elapsed, cores=1,
                distinct=len(pool))


def _oracle_worker(args):
    """One host core of the parallel oracle timing: draws its own request
    (untimed), waits for every worker, then times its share of decode steps
    on one thread."""
    wname, num_splits, n_queries, seed, barrier = args
    from threadpoolctl import threadpool_limits
    import torch
    from workloads.qsa_inputs import WORKLOADS
    torch.set_num_threads(1)
    w = WORKLOADS[wname]
    with threadpool_limits(limits=1):
        pool = oracle_pool(w, 1, seed)
        oracle_step(w, pool[0], num_splits)            # untimed warm-up
        barrier.wait()
        t0 = time.perf_counter()
        for _ in range(n_queries):
            oracle_step(w, pool[0], num_splits)
        return time.perf_counter() - t0


def host_cores(cap: int = 64) -> int:
    return max(1, min(cap, len(os.sched_getaffinity(0))))


def time_oracle_parallel(w, num_splits: int, queries_per_core: int, cores: int,
                         seed: int = 5000) -> dict:
    """Times the oracle (as it stands) on `cores` host cores at once: one
    spawn worker process per core, each running queries_per_core decode
    steps of its own drawn request on one thread, all started together after
    an untimed draw and warm-up.  value = all workers' queries / the slowest
    worker's time."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        barrier = m.Barrier(cores)
        with ctx.Pool(cores) as pool:
            times = pool.map(_oracle_worker, [(w.name, num_splits, queries_per_core,
                                               seed + 17 * i, barrier) for i in range(cores)])
    wall = max(times)
    queries = cores * queries_per_core * w.T
    return dict(value=queries / wall, queries=queries, seconds=wall, cores=cores, distinct=cores)


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from sparse_attention_decode_compress_b200 import (QSADecodeStep, qsa_get_device_error)
    from sparse_attention_decode_compress_b200 import api as qapi
    from workloads.qsa_inputs import WORKLOADS, make_batch
    sys.path.insert(0, os.path.join(ROOT, "tests"))

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    if args.batch is not None or args.ctx is not None:
        from dataclasses import replace
        w = replace(w, batch=args.batch if args.batch is not None else w.batch,
                    ctx=args.ctx if args.ctx is not None else w.ctx)
    dcp = args.dcp and world > 1
    S = world if dcp else args.splits
    # replicas draw independent batches; DCP ranks share one batch
    batch = make_batch(w, dev, seed=w.seed if dcp else rank_seed(w.seed, rank))
    B, T = w.batch, w.T
    L_host = batch.ctx_lens_host
    max_blocks = int((L_host.max() + 3) // 4)

    # caches (untimed): bulk append of all but the last T positions
    cache = qapi.QSACache.allocate(batch.k_cache, batch.v_cache, batch.block_table, w.d_idx,
                                   ring_rows=B, k_scale=batch.k_scale, v_scale=batch.v_scale)
    n_pre = (L_host - T)
    parts = [batch.k_idx[int(batch.cu_ctx_host[r]): int(batch.cu_ctx_host[r]) + int(n_pre[r])]
             for r in range(B)]
    k_pre = torch.cat(parts)
    cu_pre = torch.zeros(B + 1, dtype=torch.int32)
    cu_pre[1:] = torch.cumsum(n_pre, 0).to(torch.int32)
    qapi.qsa_compress_append(cache, torch.zeros(B, dtype=torch.int32, device=dev), cu_pre.to(dev),
                             k_pre, int(n_pre.max()))
    del k_pre, parts
    rows = torch.cat([torch.arange(int(batch.cu_ctx_host[r + 1]) - T, int(batch.cu_ctx_host[r + 1]))
                      for r in range(B)]).to(dev)
    k_new = batch.k_idx[rows].contiguous()
    cu_new = torch.arange(0, B * T + 1, T, dtype=torch.int32, device=dev)
    pos0 = (L_host - T).to(torch.int32).to(dev)
    n_sel = ((L_host - T) // 4 + 1).to(torch.int32).to(dev) if T > 1 else None
    step = QSADecodeStep(cache, B, T, w.Hq, w.topk, S, max_blocks)
    stream = torch.cuda.current_stream()
    dcp_step = None
    if dcp:
        from sparse_attention_decode_compress_b200.dcp import DCPDecode
        dcp_step = DCPDecode(cache, B, T, w.Hq, w.topk)

    def one_step(ev=None):
        qapi.qsa_compress_append(cache, pos0, cu_new, k_new, T)
        if ev is not None:
            ev[0].record(stream)
        qapi.qsa_index_topk(cache, batch.q_idx, batch.ctx_lens, n_sel, max_blocks, w.topk,
                            step.sel, None, step.ws_topk)
        if ev is not None:
            ev[1].record(stream)
        if dcp_step is not None:  # this rank's split, all-gather, merge
            dcp_step(batch.q, batch.ctx_lens, step.sel)
            if ev is not None:
                ev[2].record(stream)
            return
        qapi.qsa_sparse_decode_merged(cache, batch.q, batch.ctx_lens, step.sel, step.sm_scale, S,
                                      step.o_part, step.lse_part, step.o, step.lse, step.ws_dec)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    st, flags = qsa_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: status {st} flags {flags}")

    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    K = args.steps
    # timed region 1: K whole steps back to back (the value), as one CUDA
    # graph holding the K steps (replayed once untimed first), or as eager
    # launches with --no-graph
    graph = None
    if not args.no_graph and not dcp:  # (DCP steps hold collectives: eager)
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            for k in range(K):
                one_step()
        graph.replay()
        torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("t0")
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for k in range(K):
            one_step()
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    del graph
    # timed region 2: the same K steps with events between the kernels, for
    # the per-launch durations of the roofline (an event between two kernels
    # costs the step a few microseconds, so the value comes from region 1)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for k in range(K):
        one_step(evs[k])
    torch.cuda.synchronize()
    sampler.mark("t2")
    topk_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    st, flags = qsa_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the timed region: status {st} flags {flags}")
    ms = max_over_ranks(ms, world, dev)

    # ---- end to end through the C ABI with host buffers: the decode session
    # (qsa_session_*) uploads each step's inputs from pinned host memory and
    # downloads o / lse, overlapping the copies with the neighbouring steps
    e2e = None
    if not args.no_e2e and not dcp:
        from sparse_attention_decode_compress_b200 import QSASession
        pin = lambda t: t.cpu().pin_memory()
        h_in = dict(pos0=pin(pos0), cu_new=pin(cu_new), k_new=pin(k_new), q_idx=pin(batch.q_idx),
                    q=pin(batch.q), ctx_lens=pin(batch.ctx_lens))
        h_nsel = pin(n_sel) if n_sel is not None else None
        h2d = sum(v.numel() * v.element_size() for v in h_in.values())
        if h_nsel is not None:
            h2d += h_nsel.numel() * 4
        outs = [(torch.empty(step.o.shape, dtype=torch.float32).pin_memory(),
                 torch.empty(step.lse.shape, dtype=torch.float32).pin_memory()) for _ in range(2)]
        d2h = outs[0][0].numel() * 4 + outs[0][1].numel() * 4
        sess = QSASession(cache, B, T, w.Hq, w.topk, S, max_blocks, B * T, step.sm_scale,
                          q_dtype=batch.q.dtype, stream=stream)

        def e2e_step(k):
            o_h, lse_h = outs[k % 2]
            sess.step(h_in["pos0"], h_in["cu_new"], h_in["k_new"], h_in["q_idx"], h_in["q"],
                      h_in["ctx_lens"], h_nsel, o_h, lse_h)

        for k in range(max(3, args.warmup)):
            e2e_step(k)
        sess.synchronize()
        Ke = max(1, K // 2)
        up, _, down = sess.streams()
        s_up, s_down = torch.cuda.ExternalStream(up), torch.cuda.ExternalStream(down)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(s_up)
        for k in range(Ke):
            e2e_step(k)
        e1.record(s_down)
        sess.synchronize()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        sess.close()
        e2e = {"value": weak_scaling_rate(B * T, world, Ke, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "qsa_session_step_host (pinned host buffers, copies overlapped across steps)"}

    clocks = sampler.stop() if rank == 0 else None
    if rank != 0:
        return None

    ab = [algorithmic_bytes(w, int(L), S) for L in L_host.tolist()]
    idx_bytes = sum(a["index_topk"] for a in ab)
    tot_bytes = sum(a["total"] for a in ab)
    peaks = measured_peaks()
    queries_per_step = B * T
    # replicas: every rank runs its own batch; DCP: the ranks share one batch
    value = (weak_scaling_rate(queries_per_step, world, K, ms) if not dcp
             else queries_per_step * K / (ms / 1e3))
    hbm = (tot_bytes * K / (ms / 1e3)) / 1e9
    achieved = idx_bytes / (topk_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms / K, 5), "higher_is_better": True,
        "scaling": "strong" if dcp else "weak", "vs_baseline": None,
        "dtype": w.kv_dtype if w.kv_dtype != "f32" else "f32",
        "data": "synthetic (seeded; stands in for the pages' 256k-context serving trace)",
        "config": workload_config(w, S, world, dcp),
        "hbm_gbs": round(hbm, 1),
        "hbm_pct_of_peak": round(100 * hbm / peaks["hbm_gbs"], 2),
        "hbm_pct_of_nominal_8tbs": round(100 * hbm / 8000.0, 2),
        "roofline": {"bound": "hbm", "kernel": "index_topk", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"], "traffic": index_topk_traffic(B),
                     "launch_ms": round(topk_ms, 5), "algorithmic_bytes_per_launch": idx_bytes},
        "kernel_ms": {"index_topk": round(topk_ms, 5), "sparse_decode": round(dec_ms, 5)},
        "gpu_launches": step.kernels_per_step * K,
        "clocks": clocks,
        "e2e": e2e,
    }
    return line


PREFILL_METRIC = "QSA sparse prefill query tokens/s (chunk of the newest tokens, own selection per token)"


def prefill_flops(w, L: int, chunk: int, topk: int) -> dict:
    """Algorithmic work of a prefill chunk of one request: the indexer
    contraction (2 d int8 operations per token and competing block) and the
    attention (QK and PV: 4 D FLOPs per head and attended token)."""
    scan = att = 0
    for p in range(L - chunk, L):
        n = p // 4 + 1
        scan += 2 * w.d_idx * n
        att += 4 * w.D * w.Hq * min(4 * min(topk, n), p + 1)
    return dict(scan_int8_ops=scan, attention_flops=att)


def run_prefill(args) -> dict:
    """One step = qsa_compress_append of each request's chunk of indexer keys
    (an idempotent re-append at the same positions) + qsa_sparse_prefill of
    the chunk's tokens."""
    import torch
    from dataclasses import replace
    from sparse_attention_decode_compress_b200 import api as qapi
    from workloads.qsa_inputs import WORKLOADS, make_batch, prefill_inputs
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = replace(WORKLOADS["b32_32k"], name="prefill", batch=args.prefill_batch,
                ctx=f"fixed:{args.prefill_ctx}", planted=8,
                description=f"{args.prefill_batch} requests x {args.prefill_ctx} ctx, the newest "
                            f"{args.prefill_chunk} tokens of each as query tokens, GQA 16/2, D 128, "
                            f"bf16, page 64 random table, top-512 blocks per token")
    batch = make_batch(w, dev, seed=5)
    B, chunk = w.batch, args.prefill_chunk
    pi = prefill_inputs(batch, [chunk] * B, seed=5)
    L_host = batch.ctx_lens_host
    max_blocks = int((L_host.max() + 3) // 4)
    cache = qapi.QSACache.allocate(batch.k_cache, batch.v_cache, batch.block_table, w.d_idx,
                                   ring_rows=B)
    n_pre = L_host - chunk
    k_pre = torch.cat([batch.k_idx[int(batch.cu_ctx_host[r]): int(batch.cu_ctx_host[r]) + int(n_pre[r])]
                       for r in range(B)])
    cu_pre = torch.zeros(B + 1, dtype=torch.int32)
    cu_pre[1:] = torch.cumsum(n_pre, 0).to(torch.int32)
    qapi.qsa_compress_append(cache, torch.zeros(B, dtype=torch.int32, device=dev), cu_pre.to(dev),
                             k_pre, int(n_pre.max()))
    del k_pre
    Nq = B * chunk
    cu_q = pi["cu_q"].to(dev)
    pos0 = (L_host - chunk).to(torch.int32).to(dev)
    Hkv, D = batch.k_cache.shape[2], batch.k_cache.shape[3]
    sel = torch.empty((Nq, w.topk), dtype=torch.int32, device=dev)
    o = torch.empty((Nq, w.Hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((Nq, w.Hq), dtype=torch.float32, device=dev)
    ws = qapi.new_workspace(qapi.qsa_sparse_prefill_workspace_bytes(Nq, max_blocks, w.Hq, Hkv, D,
                                                                    w.topk), dev)
    sm = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream()

    def one_step(ev=None):
        qapi.qsa_compress_append(cache, pos0, cu_q, pi["k_chunk"], chunk)
        if ev is not None:
            ev[0].record(stream)
        qapi.qsa_sparse_prefill(cache, cu_q, batch.ctx_lens, chunk, pi["q_idx"], pi["k_chunk"],
                                pi["q"], max_blocks, w.topk, sm, sel, o, lse, ws)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    st, flags = qapi.qsa_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: status {st} flags {flags}")
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    K = args.steps
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        for _ in range(K):
            one_step()
    graph.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark("t0")
    t0.record(stream)
    graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    ms = t0.elapsed_time(t1)
    del graph
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    for k in range(K):
        one_step(evs[k])
    torch.cuda.synchronize()
    sampler.mark("t2")
    pre_ms = sum(a.elapsed_time(b) for a, b in evs) / K
    st, flags = qapi.qsa_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the timed region: status {st} flags {flags}")
    clocks = sampler.stop()
    peaks = measured_peaks()
    f = [prefill_flops(w, int(L), chunk, w.topk) for L in L_host.tolist()]
    att = sum(x["attention_flops"] for x in f)
    scan = sum(x["scan_int8_ops"] for x in f)
    # bf16-equivalent work: int8 tensor-core operations run at twice the
    # bf16 rate (nominal 4.5 vs 2.25 PFLOP/s dense)
    work = att + scan / 2
    achieved = work / (pre_ms / 1e3) / 1e12
    return {
        "metric": PREFILL_METRIC, "value": round(Nq * K / (ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded)",
        "config": {"workload": "prefill", "description": w.description, "global_batch": B,
                   "seq_len": args.prefill_ctx, "query_tokens": chunk, "topk_blocks": w.topk,
                   "page_size": w.page_size, "parallelism": "single GPU",
                   "timing": "value: K steps (append + prefill) as one CUDA graph replay; "
                             "roofline: eager pass with events around the prefill call"},
        "roofline": {"bound": "tensor", "kernel": "qsa_sparse_prefill (all its kernels)",
                     "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "peak_source": peaks["source"], "traffic": None,
                     "launch_ms": round(pre_ms, 5),
                     "flops_per_launch": {"attention": att, "scan_int8_ops": scan}},
        "gpu_launches": 6 * K,
        "clocks": clocks,
    }


def main(argv=None):
    args = parse_args(argv)
    if args.prefill and args.impl == "ours":
        print(json.dumps(run_prefill(args)), flush=True)
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        from workloads.qsa_inputs import WORKLOADS
        w = WORKLOADS[args.workload]
        # a step: one decode query of the workload on every host core (the
        # warm-up steps run untimed inside each worker)
        cores = host_cores()
        res = time_oracle_parallel(w, args.splits, args.steps, cores, seed=3000)
        line = {"metric": METRIC, "value": round(res["value"], 4), "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * res["seconds"] / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
                "data": "synthetic (seeded; stands in for the pages' 256k-context serving trace)",
                "config": workload_config(w, args.splits, max(1, args.gpus)),
                "cpu_baseline": {"value": round(res["value"], 4), "unit": UNIT, "cores": res["cores"],
                                 "kind": "oracle",
                                 "sample": f"{args.steps} decode steps of {args.workload} on each of "
                                           f"{res['cores']} host cores (one drawn request per "
                                           f"core), NumPy oracle, one thread per core"},
                "e2e": {"value": round(res["value"], 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    line = run_ours(args, rank, world, local_rank)
    if rank == 0 and line is not None:
        if not args.no_cpu_baseline and world == 1:  # the host baseline: one GPU runs only
            from workloads.qsa_inputs import WORKLOADS
            w = WORKLOADS[args.workload]
            one = time_oracle(w, args.splits, args.cpu_queries)
            cores = host_cores()
            per_core = max(1, args.cpu_queries // 10)
            res = time_oracle_parallel(w, args.splits, per_core, cores)
            line["cpu_baseline"] = {"value": round(res["value"], 4), "unit": UNIT, "cores": res["cores"],
                                    "kind": "oracle",
                                    "sample": f"{per_core} decode steps of {args.workload} on each "
                                              f"of {res['cores']} host cores (one drawn request "
                                              f"per core, one thread each), NumPy oracle, "
                                              f"{res['seconds']:.1f} s",
                                    "value_1core": round(one["value"], 4),
                                    "sample_1core": f"{one['queries']} decode steps (cycling over "
                                                    f"{one['distinct']} drawn requests) on 1 host "
                                                    f"core, {one['seconds']:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
