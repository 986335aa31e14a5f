"""Throughput of the FBNL scoring path: reranked pairs/s on one query of 100 documents (Nano shape).

python bench.py [--gpus N] [--steps K] [--warmup W] [--config nano] [--impl kalm|reference]

One step = one query through the whole path (chunk pooling of every document's
encoder states, the cross K/V projection of all layers, 18 decoder layers of
Q|K|V projection + merged attention + output projection, and the yes/no
readout), replayed as one CUDA graph with every input resident in HBM.  The L2
is flushed (a 256 MiB write) before every step, outside the step's CUDA-event
interval.  Rank 0 prints one JSON line.

Multi-GPU (torchrun): every rank scores its own query of the same shape (the
path shards by documents and queries; nothing crosses GPUs on the data path),
so per-GPU work is fixed ("weak" scaling).  Timing is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this path has)
on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "reranked pairs/s (Nano shape, 1 B200); pool GB/s and attn TFLOP/s vs peak"
UNIT = "pairs/s"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="nano", choices=["tiny", "nano", "small", "large"])
    ap.add_argument("--impl", default="kalm", choices=["kalm", "reference"])
    ap.add_argument("--cpu-sample-docs", type=int, default=0, help="documents in the oracle sample (0 = auto)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-pool-sweep", action="store_true", help="skip the pooling-only sweep at 1024/4096 docs")
    ap.add_argument("--no-fused", action="store_true", help="skip the fused attention + output projection step")
    ap.add_argument("--no-chain", action="store_true",
                    help="run each output projection and the next Q|K|V projection as two launches")
    ap.add_argument("--rope-theta", type=float, default=None,
                    help="rotate the decoder's self Q/K with this rotary base in every layer (default: off)")
    ap.add_argument("--sweep", action="store_true",
                    help="end-to-end throughput at the sweep shapes (1..4096 documents per query), one JSON line")
    ap.add_argument("--pool-sweep-only", action="store_true",
                    help="run only the pooling sweep at 1024/4096 documents and print it as one JSON line")
    return ap.parse_args()


def traffic(label: str):
    """DRAM bytes per launch of a kernel from profiles/dram_traffic.txt, or None if its
    sources changed since the capture (the counters no longer describe this kernel)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        k, b, digest, srcs = line.split()
        if k != label:
            continue
        h = hashlib.sha256()
        for src in srcs.split(","):
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        return int(b) if h.hexdigest()[:16] == digest else None
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# algorithmic work (what the method must do; padding and masked keys not counted)
# ---------------------------------------------------------------------------
def workload(q, chain: bool = True):
    """Algorithmic work of one step, per kernel kind (summed over its launches), for
    the pruned layer stack the scorer runs: the first layer's Q|K|V projection on
    the query's common input only, and in the last layer attention for the query
    tile holding each document's final row and the output projection of that row.
    With ``chain`` (the scorer's default) every other layer's output projection and
    the next layer's Q|K|V projection are one launch, labelled o_proj_qkv."""
    H, D, nq, nkv, L, lq = q.hidden, q.head_dim, q.n_q, q.n_kv, q.layers, q.lq
    n = q.n_docs
    lens = q.doc_len.astype(np.int64)
    nc = (lens + 3) // 4
    rows = n * lq
    G = nq // nkv
    P = 128 // G
    w = {}
    w["pool_bytes"] = int((lens.sum() + nc.sum()) * H * 2 + 8 * n)
    w["cross_kv_proj"] = int(2 * nc.sum() * H * 2 * nkv * D * L)
    qkv_row = 2 * H * (nq + 2 * nkv) * D
    w["qkv_proj"] = int(qkv_row * (lq + rows * (L - 1)))
    full_attn = 4 * nq * D * (n * lq * (lq + 1) // 2 + lq * int(nc.sum()))
    t_last = (lq - 1) // P
    last_rows = np.arange(t_last * P, lq)
    last_attn = 4 * nq * D * (n * int((last_rows + 1).sum()) + len(last_rows) * int(nc.sum()))
    w["merged_attention"] = int(full_attn * (L - 1) + last_attn)
    w["o_proj"] = int(2 * nq * D * H * (rows * (L - 1) + n))
    w["total_flops"] = w["cross_kv_proj"] + w["qkv_proj"] + w["merged_attention"] + w["o_proj"]
    # unfused algorithmic bytes (each operand read once, each result written once), for the
    # arithmetic-intensity bound min(peak, AI * HBM)
    P_ = int(nc.sum())
    w["bytes"] = {
        "cross_kv_proj": 2 * (P_ * H + L * 2 * nkv * D * H + P_ * L * 2 * nkv * D),
        "qkv_proj": 2 * ((lq + rows * (L - 1)) * (H + (nq + 2 * nkv) * D) + L * (nq + 2 * nkv) * D * H),
        "merged_attention": 2 * (L - 1) * (rows * (2 * nq + 2 * nkv) * D + P_ * 2 * nkv * D)
                            + 2 * (n * P * 2 * nq * D + rows * 2 * nkv * D + P_ * 2 * nkv * D),
        "o_proj": 2 * ((rows * (L - 1) + n) * (nq * D + 2 * H) + L * H * nq * D),
    }
    if chain and L > 1:
        # the chained launches: output projections of layers 0 .. L-2 (with the residual)
        # and Q|K|V projections of layers 1 .. L-1, each operand read once and each
        # result written once
        w["o_proj_qkv"] = int(2 * nq * D * H * rows * (L - 1) + qkv_row * rows * (L - 1))
        w["qkv_proj"] = int(qkv_row * lq)
        w["o_proj"] = int(2 * nq * D * H * n)
        w["bytes"]["o_proj_qkv"] = 2 * ((L - 1) * rows * (nq * D + 2 * H) + (L - 1) * H * nq * D
                                        + (L - 1) * rows * (H + (nq + 2 * nkv) * D) + (L - 1) * (nq + 2 * nkv) * D * H)
        w["bytes"]["qkv_proj"] = 2 * (lq * (H + (nq + 2 * nkv) * D) + (nq + 2 * nkv) * D * H)
        w["bytes"]["o_proj"] = 2 * (n * (nq * D + 2 * H) + H * nq * D)
    return w


def pool_chunks(enc, len_d, chunks=(1, 2, 4, 8), reps=10):
    """The pooling kernel alone on one query's encoder states at each chunk size
    (Matryoshka granularities): median time of `reps` calls with the L2 flushed before
    each (CUDA events), algorithmic bytes, GB/s."""
    import torch
    from encoder_decoder_document_b200 import kalm_chunk_pool, kalm_ragged_offsets
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    n, H = len_d.numel(), enc.shape[1]
    lens = len_d.cpu().numpy().astype(np.int64)
    out = []
    for c in chunks:
        nc = (lens + c - 1) // c
        tok_off = torch.empty(n + 1, dtype=torch.int64, device="cuda")
        pool_off = torch.empty(n + 1, dtype=torch.int64, device="cuda")
        kalm_ragged_offsets(len_d, tok_off, pool_off, c)
        pooled = torch.empty(int(nc.sum()), H, dtype=torch.bfloat16, device="cuda")
        ts = []
        for i in range(reps + 2):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            kalm_chunk_pool(enc, tok_off, len_d, pooled, pool_off, pooled.shape[0], c)
            b.record()
            b.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b))
        us = 1e3 * statistics.median(ts)
        byts = int((lens.sum() + nc.sum()) * H * 2 + 8 * n)
        out.append({"chunk": c, "bytes": byts, "us": us, "gbs": byts / (us * 1e-6) / 1e9})
    return out


def fused_layers(args, q, weights_dev, w, pk):
    """The same query through a scorer whose layers (all but the pruned last one) run as
    one fused attention + output projection launch (kalm_merged_attention_out_proj):
    steps of its graph timed like the main step (L2 flushed before each), and the fused
    kernel's own launch time from its instrumented graph."""
    import torch
    from encoder_decoder_document_b200.scorer import FBNLScorer
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    sc = FBNLScorer(weights_dev, q.n_q, q.n_kv, rope_theta=args.rope_theta, fused_out=True)
    total_pooled = int(((q.doc_len.astype(np.int64) + 3) // 4).sum())
    sc.prepare(q.n_docs, int(q.doc_len.sum()), total_pooled, q.lq)
    sc.load_inputs(torch.from_numpy(q.enc.view(np.int16)).view(torch.bfloat16), torch.from_numpy(q.doc_len),
                   torch.from_numpy(q.x0.view(np.int16)).view(torch.bfloat16))
    sc.capture(instrument=True)
    step_ms, per = [], {}
    for i in range(max(args.warmup, 3) + args.steps):
        for g in (sc.graph, sc.graph_inst):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            if i >= max(args.warmup, 3):
                if g is sc.graph:
                    step_ms.append(a.elapsed_time(b))
                else:
                    for label, v in sc.kernel_times().items():
                        per.setdefault(label, []).extend(v)
    from encoder_decoder_document_b200 import kalm_check_device_errors
    kalm_check_device_errors()
    ms = sum(step_ms) / len(step_ms)
    fused_us = 1e3 * statistics.mean(per["attention_out_proj"])
    n_fused = len(per["attention_out_proj"]) / args.steps
    # algorithmic FLOPs of one fused launch: a full layer's attention and output projection
    H, D, nq, lq, n = q.hidden, q.head_dim, q.n_q, q.lq, q.n_docs
    nc = int(((q.doc_len.astype(np.int64) + 3) // 4).sum())
    flops = 4 * nq * D * (n * lq * (lq + 1) // 2 + lq * nc) + 2 * nq * D * H * n * lq
    out = {"value": q.n_docs / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "launches_per_step": n_fused,
           "fused_avg_us": fused_us, "fused_tflops": flops / (fused_us * 1e-6) / 1e12,
           "fused_frac": flops / (fused_us * 1e-6) / 1e12 / pk["bf16"],
           "how": "FBNLScorer(fused_out=True): merged attention and output projection + residual of every layer "
                  "but the last in one persistent launch; projection tiles claimed as CTAs finish their attention "
                  "items, each waiting only for its own document"}
    del sc
    return out


def plain_copy(src, reps=10):
    """A plain device copy (torch) of the encoder states the pooling reads, L2 flushed
    before each call: the bandwidth a read of that size reaches without any pooling
    (bytes = read + write of the tensor)."""
    import torch
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    dst = torch.empty_like(src)
    ts = []
    for i in range(reps + 2):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src)
        b.record()
        b.synchronize()
        if i >= 2:
            ts.append(a.elapsed_time(b))
    us = 1e3 * statistics.median(ts)
    byts = 2 * src.numel() * src.element_size()
    return {"bytes": byts, "us": us, "gbs": byts / (us * 1e-6) / 1e9}


def rope_alone(sc, theta=1e4, reps=10):
    """Cost of the rotary embedding on one layer's Q|K|V (all documents' rows, Q and
    self-K heads), L2 flushed before each call, medians: the standalone rotation
    kernel (bytes read + written, GB/s), and the Q|K|V projection without and with
    the rotation fused into its epilogue."""
    import torch
    from encoder_decoder_document_b200 import kalm_linear, kalm_linear_rope, kalm_rope, kalm_rope_table
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    heads = sc.n_q + sc.n_kv
    w = sc.w.w_qkv[1]

    def timed(fn):
        ts = []
        for i in range(reps + 2):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b))
        return 1e3 * statistics.median(ts)

    us = timed(lambda: kalm_rope(sc.qkv, sc.q_off, heads, theta, sc.D))
    plain = timed(lambda: kalm_linear(sc.x, w, sc.qkv))
    table = kalm_rope_table(theta, sc.D)
    fused = timed(lambda: kalm_linear_rope(sc.x, w, sc.qkv, sc.q_off, heads, table, sc.D))
    byts = 2 * sc.qkv.shape[0] * heads * sc.D * 2
    return {"rows": sc.qkv.shape[0], "heads": heads, "theta": theta, "bytes": byts, "us": us,
            "gbs": byts / (us * 1e-6) / 1e9, "qkv_proj_us": plain, "qkv_proj_rope_us": fused,
            "fused_extra_us": fused - plain}


def sweep_queries(n_docs: int) -> int:
    """Distinct queries timed per sweep point (the configuration names 1,000 per point;
    a bounded number keeps the run within minutes): 8, and 2 at 4096 documents."""
    return 8 if n_docs <= 1024 else 2


def run_sweep(args, doc_counts=(1, 16, 100, 1024, 4096)):
    """End-to-end throughput at the sweep shapes (Nano model, log-normal lengths with
    median 200 clipped to [1, 1024], Lq drawn from [32, 512] per query): at each point,
    distinct seeded queries (seed 4 + k for query k), each with its own lengths, its own
    query length and its own captured graph; K steps per query, L2 flushed before each
    step.  Per point: total documents / total time over its queries, plus the pooling and
    attention kernels' own times from each query's instrumented graph, and (unless the CPU
    baseline is switched off) the oracle timed on two documents of the point's first query."""
    import torch
    import synthetic
    from encoder_decoder_document_b200 import _build, kalm_check_device_errors
    from encoder_decoder_document_b200.scorer import DeviceWeights, FBNLScorer
    _build.build()
    pk = peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    weights = synthetic.make_query("sweep", n_docs=1, seed=4).weights
    dw = DeviceWeights.from_bits(weights)
    out = []
    for n in doc_counts:
        nq = sweep_queries(n)
        tot_ms, tot_docs, lqs = 0.0, 0, []
        attn_us, attn_flops, pool_us, pool_bytes, flops = 0.0, 0, 0.0, 0, 0
        oracle_cb = None
        for k in range(nq):
            q = synthetic.make_query("sweep", n_docs=n, seed=4 + k, with_weights=False)
            q = dataclasses.replace(q, weights=weights)
            if k == 0 and not args.no_cpu_baseline:
                oracle_cb = cpu_baseline(q, min(2, n))
            sc = FBNLScorer(dw, q.n_q, q.n_kv, chain=not args.no_chain)
            w = workload(q, chain=sc.chain)
            total_pooled = int(((q.doc_len.astype(np.int64) + 3) // 4).sum())
            sc.prepare(q.n_docs, int(q.doc_len.sum()), total_pooled, q.lq)
            sc.load_inputs(torch.from_numpy(q.enc.view(np.int16)).view(torch.bfloat16),
                           torch.from_numpy(q.doc_len), torch.from_numpy(q.x0.view(np.int16)).view(torch.bfloat16))
            sc.capture(instrument=True)
            ts, per = [], {}
            for i in range(args.warmup + args.steps):
                for g in (sc.graph, sc.graph_inst):
                    flush.fill_(1.0)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    g.replay()
                    b.record()
                    b.synchronize()
                    if i >= args.warmup:
                        if g is sc.graph:
                            ts.append(a.elapsed_time(b))
                        else:
                            for label, v in sc.kernel_times().items():
                                per.setdefault(label, []).extend(v)
            kalm_check_device_errors()
            tot_ms += sum(ts)
            tot_docs += n * len(ts)
            lqs.append(q.lq)
            attn_us += 1e3 * sum(per["merged_attention"]) / args.steps
            attn_flops += w["merged_attention"]
            pool_us += 1e3 * statistics.mean(per["chunk_pool"])
            pool_bytes += w["pool_bytes"]
            flops += w["total_flops"] * len(ts)
            del sc
        torch.cuda.empty_cache()
        out.append({"docs": n, "queries": nq, "steps_per_query": args.steps, "lq": lqs,
                    "ms_per_query": tot_ms * n / tot_docs, "pairs_per_s": tot_docs / (tot_ms * 1e-3),
                    "step_tflops": flops / (tot_ms * 1e-3) / 1e12,
                    "attention_us_per_query": attn_us / nq, "attention_tflops": attn_flops / (attn_us * 1e-6) / 1e12,
                    "pool_us_per_query": pool_us / nq, "pool_gbs": pool_bytes / (pool_us * 1e-6) / 1e9,
                    "pool_frac": pool_bytes / (pool_us * 1e-6) / 1e9 / pk["hbm"],
                    "cpu_baseline": oracle_cb})
        print(json.dumps(out[-1]), flush=True)
    return out


def pool_sweep(doc_counts=(1024, 4096), reps=10):
    """The pooling kernel alone at the throughput-sweep shapes with many documents
    (hidden 640, log-normal lengths, median 200, clipped to [1, 1024]): bytes moved,
    median time of `reps` calls (L2 flushed before each, CUDA events), GB/s."""
    import torch
    import synthetic
    from encoder_decoder_document_b200 import kalm_chunk_pool, kalm_ragged_offsets
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    gen = torch.Generator(device="cuda")
    out = []
    for n in doc_counts:
        lens = synthetic.draw_lengths(synthetic.CONFIGS["sweep"]["len"], n, np.random.default_rng([4, n]))
        H = synthetic.CONFIGS["sweep"]["hidden"]
        total = int(lens.sum())
        nc = (lens.astype(np.int64) + 3) // 4
        gen.manual_seed(4 * 100003 + n)
        enc = torch.randn(total, H, device="cuda", generator=gen).to(torch.bfloat16)
        len_d = torch.from_numpy(lens).cuda()
        tok_off = torch.empty(n + 1, dtype=torch.int64, device="cuda")
        pool_off = torch.empty(n + 1, dtype=torch.int64, device="cuda")
        kalm_ragged_offsets(len_d, tok_off, pool_off, 4)
        pooled = torch.empty(int(nc.sum()), H, dtype=torch.bfloat16, device="cuda")
        ts = []
        for i in range(reps + 2):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            kalm_chunk_pool(enc, tok_off, len_d, pooled, pool_off, pooled.shape[0], 4)
            b.record()
            b.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b))
        us = 1e3 * statistics.median(ts)
        byts = int((total + int(nc.sum())) * H * 2 + 8 * n)
        out.append({"docs": n, "encoder_tokens": total, "bytes": byts, "us": us, "gbs": byts / (us * 1e-6) / 1e9})
        del enc, pooled
    return out


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


def cpu_baseline(q, n_sample: int, one_thread_docs: int = 0):
    """The fp64 oracle (as it stands: a per-document loop whose matrix products run on
    the BLAS thread pool) on the first n_sample documents of the query.  ``cores`` is
    the BLAS pool's thread count, the threads the oracle actually used; ``host_cores``
    the host's logical CPUs.  With ``one_thread_docs`` the same oracle is also timed
    with the BLAS pool limited to one thread on that many documents."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    t0 = time.perf_counter()
    oracle.forward_query(q, docs=range(n_sample))
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    res = {"value": n_sample / dt, "unit": UNIT, "cores": threads, "host_cores": os.cpu_count(), "kind": "oracle",
           "sample": f"{n_sample} of {q.n_docs} documents of one {q.name} query, all {q.layers} layers, fp64 "
                     f"numpy, documents one after another, matrix products on {threads} BLAS threads; {dt:.1f} s"}
    if one_thread_docs:
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            oracle.forward_query(q, docs=range(one_thread_docs))
            dt1 = time.perf_counter() - t0
        res["one_thread"] = {"value": one_thread_docs / dt1, "unit": UNIT, "cores": 1,
                             "sample": f"{one_thread_docs} documents, BLAS limited to 1 thread; {dt1:.1f} s"}
    return res


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synthetic
    q = synthetic.make_query(args.config)
    n_sample = args.cpu_sample_docs or (2 if args.config in ("nano", "tiny") else 1)
    n_sample = min(n_sample, q.n_docs)
    for _ in range(args.warmup):
        cpu_baseline(q, 1)
    times = []
    cb = None
    for _ in range(args.steps):
        cb = cpu_baseline(q, n_sample)
        times.append(n_sample / cb["value"])
    total = sum(times)
    value = n_sample * args.steps / total
    cb["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{q.name}: 1 query x {n_sample} sampled documents per step (of {q.n_docs})",
                       "hidden": q.hidden, "layers": q.layers, "lq": q.lq},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.sweep:
        print(json.dumps({"sweep": run_sweep(args)}), flush=True)
        return
    if args.pool_sweep_only:
        pk = peaks()
        sweep = [dict(x, peak_gbs=pk["hbm"], frac=x["gbs"] / pk["hbm"]) for x in pool_sweep()]
        print(json.dumps({"pool_sweep": sweep}), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import synthetic
    from encoder_decoder_document_b200 import _build, kalm_check_device_errors
    from encoder_decoder_document_b200.scorer import DeviceWeights, FBNLScorer

    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    # each rank scores its own query (its own document shard) of the configured shape
    base = synthetic.CONFIGS[args.config]["seed"]
    q = synthetic.make_query(args.config, seed=base if rank == 0 else base + 1000 * rank)
    pk = peaks()
    sc = FBNLScorer(DeviceWeights.from_bits(q.weights), q.n_q, q.n_kv, rope_theta=args.rope_theta,
                    chain=not args.no_chain)
    w = workload(q, chain=sc.chain)
    total_pooled = int(((q.doc_len.astype(np.int64) + 3) // 4).sum())
    sc.prepare(q.n_docs, int(q.doc_len.sum()), total_pooled, q.lq)
    enc_h = torch.from_numpy(q.enc.view(np.int16)).view(torch.bfloat16).pin_memory()
    len_h = torch.from_numpy(q.doc_len).pin_memory()
    x0_h = torch.from_numpy(q.x0.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_h = torch.empty(4, q.n_docs, dtype=torch.float32).pin_memory()
    sc.load_inputs(enc_h, len_h, x0_h)
    sc.capture(instrument=True)
    launches_per_step = sc.launches
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def step_timed(graph):
        flush.fill_(1.0)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        return a, b

    for _ in range(max(args.warmup, 3)):
        step_timed(sc.graph)
        step_timed(sc.graph_inst)
    torch.cuda.synchronize()
    kalm_check_device_errors()

    # ---------------- timed region: K steps of the plain graph (the step time), each
    # followed by one replay of the instrumented graph (per-kernel durations)
    clocks = Clocks(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    step_ms = []
    per_kernel: dict = {}
    for _ in range(args.steps):
        a, b = step_timed(sc.graph)
        b.synchronize()
        step_ms.append(a.elapsed_time(b))
        _, bi = step_timed(sc.graph_inst)
        bi.synchronize()
        for label, v in sc.kernel_times().items():
            per_kernel.setdefault(label, []).extend(v)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    kalm_check_device_errors()
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], device="cuda", dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * q.n_docs * args.steps / (total_ms / 1e3)

    # ---------------- end to end through the public API: every step copies its inputs
    # host -> device (pinned) and reads its scores back.  Pipelined: FBNLScorer.score_stream
    # copies query k+1 while query k runs (the serving path); serial: copy, run, read back.
    n_e2e = args.steps
    outs = [torch.empty(4, q.n_docs, dtype=torch.float32).pin_memory() for _ in range(2)]
    inputs = [(enc_h, len_h, x0_h)] * n_e2e
    sc.score_stream(inputs[: max(args.warmup, 3)], [outs[k % 2] for k in range(max(args.warmup, 3))])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    sc.score_stream(inputs, [outs[k % 2] for k in range(n_e2e)])
    b.record(stream)
    b.synchronize()
    e2e_total = a.elapsed_time(b)
    serial_ms = []
    for _ in range(max(args.warmup, 3) + args.steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sc.load_inputs(enc_h, len_h, x0_h)
        sc.graph.replay()
        sc.scores_to_host(out_h)
        b.record(stream)
        b.synchronize()
        serial_ms.append(a.elapsed_time(b))
    serial_total = sum(serial_ms[max(args.warmup, 3):])

    # ---------------- persistent-cache regime: the same documents against many queries; the
    # documents' pooled vectors and cross K/V are built once, each query runs the decoder only
    sc.cache_documents(enc_h, len_h)
    dec_graph = sc.graphs_decode[sc.slot]
    dec_ms = []
    for i in range(max(args.warmup, 3) + args.steps):
        a, b = step_timed(dec_graph)
        b.synchronize()
        if i >= max(args.warmup, 3):
            dec_ms.append(a.elapsed_time(b))
    x0s = [x0_h] * n_e2e
    sc.score_cached_stream(x0s[: max(args.warmup, 3)], [outs[k % 2] for k in range(max(args.warmup, 3))])
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    sc.score_cached_stream(x0s, [outs[k % 2] for k in range(n_e2e)])
    b.record(stream)
    b.synchronize()
    dec_e2e_total = a.elapsed_time(b)
    dec_total = sum(dec_ms)
    if world > 1:
        t = torch.tensor([e2e_total, serial_total, dec_total, dec_e2e_total], device="cuda", dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_total, serial_total, dec_total, dec_e2e_total = (float(x) for x in t.tolist())
    kalm_check_device_errors()
    h2d = enc_h.numel() * 2 + len_h.numel() * 4 + x0_h.numel() * 2
    d2h = out_h.numel() * 4

    # ---------------- per-kernel summary and roofline of the dominant kernel
    kern = {}
    grand = max(sum(sum(x) for x in per_kernel.values()), 1e-12)
    for label, v in per_kernel.items():
        kern[label] = {"launches_per_step": len(v) / args.steps, "avg_us": 1e3 * statistics.mean(v),
                       "us_per_step": 1e3 * sum(v) / args.steps, "share": sum(v) / grand}
    tensor_kernels = [k for k in kern if k in ("qkv_proj", "o_proj", "o_proj_qkv", "merged_attention", "cross_kv_proj")]
    for k in tensor_kernels:
        kern[k]["tflops"] = w[k] / (kern[k]["us_per_step"] * 1e-6) / 1e12
    dom = max(tensor_kernels, key=lambda k: kern[k]["share"])
    dom_ach = kern[dom]["tflops"]
    ai = w[dom] / w["bytes"][dom]
    ai_bound = min(pk["bf16"], ai * pk["hbm"] / 1e3)
    roofline = {"kernel": dom, "bound": "tensor", "achieved": dom_ach, "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": dom_ach / pk["bf16"], "traffic": traffic(dom),
                "peak_source": f"{pk['source']} dense bf16 burst (cuBLAS), of measured",
                "frac_sustained": dom_ach / pk["bf16_sustained"], "peak_sustained": pk["bf16_sustained"],
                "ai_flop_per_byte": ai, "ai_bound": ai_bound, "frac_of_ai_bound": dom_ach / ai_bound}
    for k in tensor_kernels:
        ai_k = w[k] / w["bytes"][k]
        kern[k]["frac_burst"] = kern[k]["tflops"] / pk["bf16"]
        kern[k]["frac_sustained"] = kern[k]["tflops"] / pk["bf16_sustained"]
        kern[k]["ai_flop_per_byte"] = ai_k
        kern[k]["frac_of_ai_bound"] = kern[k]["tflops"] / min(pk["bf16"], ai_k * pk["hbm"] / 1e3)
    pool_gbs = w["pool_bytes"] / (kern["chunk_pool"]["avg_us"] * 1e-6) / 1e9
    copy_ref = plain_copy(sc.enc[: int(q.doc_len.sum())])
    attn_proj_us = sum(kern[k]["us_per_step"] for k in ("merged_attention", "cross_kv_proj") if k in kern)
    attn_proj_flops = w["cross_kv_proj"] + w["merged_attention"]
    step_flops = w["total_flops"]
    ms_step = total_ms / args.steps

    if rank == 0:
        cb = None
        sweep = None if args.no_pool_sweep else [dict(x, peak_gbs=pk["hbm"], frac=x["gbs"] / pk["hbm"])
                                                 for x in pool_sweep()]
        chunks = None if args.no_pool_sweep else [dict(x, frac=x["gbs"] / pk["hbm"])
                                                  for x in pool_chunks(sc.enc[: int(q.doc_len.sum())], sc.doc_len)]
        rope = None if args.no_pool_sweep else dict(rope_alone(sc), frac=None)
        fused = None if (args.no_fused or world > 1) else fused_layers(args, q, sc.w, w, pk)
        if rope is not None:
            rope["frac"] = rope["gbs"] / pk["hbm"]
        if not args.no_cpu_baseline and world == 1:
            n_cpu = min(args.cpu_sample_docs or q.n_docs, q.n_docs)
            cb = cpu_baseline(q, n_cpu, one_thread_docs=min(10, n_cpu))
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{q.name}: 1 query x {q.n_docs} documents per GPU, hidden {q.hidden}, "
                                   f"Lq {q.lq}, {q.n_q}q/{q.n_kv}kv heads x 256, {q.layers} layers",
                       "docs_per_step": q.n_docs * world, "encoder_tokens": int(q.doc_len.sum()),
                       "pooled_vectors": total_pooled, "parallelism": f"dp{world} (independent queries)",
                       "l2": "flushed (256 MiB write) before every step, outside the step's events",
                       "graph": "one CUDA graph per step (launches overlap through programmatic dependent "
                                "launch); per-kernel times come from a second graph with a timing event "
                                "after every launch, replayed once after each timed step",
                       "instrumented_ms_per_step": sum(sum(v) for v in per_kernel.values()) / args.steps,
                       "rope_theta": args.rope_theta},
            "roofline": roofline,
            "algorithmic_flops_per_step": step_flops,
            "pool": {"bytes": w["pool_bytes"], "avg_us": kern["chunk_pool"]["avg_us"], "achieved_gbs": pool_gbs,
                     "peak_gbs": pk["hbm"], "frac": pool_gbs / pk["hbm"],
                     "plain_copy_same_size": dict(copy_ref, frac=copy_ref["gbs"] / pk["hbm"]),
                     "frac_of_plain_copy": pool_gbs / copy_ref["gbs"]},
            "attn_plus_cross_proj": {"flops": attn_proj_flops, "us": attn_proj_us,
                                     "tflops": attn_proj_flops / (attn_proj_us * 1e-6) / 1e12,
                                     "frac": attn_proj_flops / (attn_proj_us * 1e-6) / 1e12 / pk["bf16"]},
            "step_tflops": step_flops / (ms_step * 1e-3) / 1e12,
            "kernels": kern,
            "e2e": {"value": world * q.n_docs * n_e2e / (e2e_total / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_total / n_e2e,
                    "how": "FBNLScorer.score_stream over K queries: pinned host inputs copied to the device and "
                           "scores read back every step; query k+1's copy overlaps query k's compute",
                    "serial": {"value": world * q.n_docs * args.steps / (serial_total / 1e3),
                               "ms_per_step": serial_total / args.steps,
                               "how": "copy in, replay, copy out, one step at a time"}},
            "decode_only": {"value": world * q.n_docs * args.steps / (dec_total / 1e3), "unit": UNIT,
                            "ms_per_step": dec_total / args.steps,
                            "e2e": {"value": world * q.n_docs * n_e2e / (dec_e2e_total / 1e3), "unit": UNIT,
                                    "h2d_bytes_per_step": x0_h.numel() * 2, "d2h_bytes_per_step": d2h},
                            "how": "persistent-cache regime: the documents' pooled vectors and every layer's cross "
                                   "K/V built once (FBNLScorer.cache_documents); each step is one query through "
                                   "the decoder-only graph (L2 flushed before each step); e2e through "
                                   "FBNLScorer.score_cached_stream with the query input copied in and scores read "
                                   "back"},
            "fused_layer": fused,
            "pool_sweep": sweep,
            "pool_chunks": chunks,
            "rope": rope,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "cpu_baseline": cb,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        sc.graph = None
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
