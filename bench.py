#!/usr/bin/env python
"""Decode benchmark of the ZHA hot path on B200.

Workload (default): the 256K-context deep-tree decode run -- 8 sequences, 16
query / 2 KV heads, d = 128, 262,144 cached tokens, tree of blocks of 4 over 6
levels, p = 0.95. One step appends one token per sequence and runs
zha_extend_tree + the traversal + sparse attention for all 128 (sequence,
head) queries. Inputs are synthetic (seeded Gaussian-mixture keys with planted
needles) and resident in HBM; K+V (2.15 GB) is larger than L2, so no flush is
needed between steps.

--workload prefill-deep-1m-chunk4k times chunked prefill instead: a 4096-token
chunk (16 query / 2 KV heads) after 1,048,576 cached tokens, one step being
zha_prefill_chunk over the whole chunk (tree extension, tensor-core top level
with certificates, traversal and sparse attention for all 65,536 queries).
The default decode line also carries a short run of it (`prefill_chunk`), as
well as the wide-tree p sweep and the other workloads' tree builds.

One JSON line on rank 0. Under torchrun every rank runs an independent replica
(weak scaling, no data-path collective); timing is the max over ranks.
--impl reference times the CPU oracle on the same metric (a bounded sample).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

WORKLOAD = "decode-deep-256k-b8"
METRIC = "ZHA decode queries/s at 256K ctx (B=8, p=0.95); % of HBM roofline"
PREFILL_METRIC = "ZHA chunked-prefill queries/s (4096-token chunk after 1M tokens, p=0.95)"


def is_prefill(name: str) -> bool:
    return name.startswith("prefill")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="zha", choices=["zha", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--n-tokens", type=int, default=None,
                    help="context length override (profiling captures on a smaller case); "
                         "the reported workload is the full one only without it")
    ap.add_argument("--sweep", action="store_true",
                    help="tree-geometry sweep of the decode workload (one JSON line per "
                         "geometry): selectivity and queries/s against the dense kernel")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait(timeout=5)
        self.thread.join(timeout=5)  # the reader drains stdout to its end first
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def strip_c_comments(src: str) -> str:
    """C/C++ source without its comments, each whitespace run folded to one
    space; string and character literals are kept as written."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def prefill_selection(lc, b: int, L: int, start: int) -> dict:
    """Per-query selection figures of a prefill chunk from kept counts lc
    [T][Hq][L] (top level first), token i of the chunk at position start + i:
    the mean kept nodes per level, and the mean fraction of the t + 1 visible
    tokens a query at t selects -- b per kept level-1 node plus the tail past
    its last complete top node (token 0 adds at most one more)."""
    T = lc.shape[0]
    vis = torch.arange(start + 1, start + T + 1, dtype=torch.int64)  # t + 1
    tail = vis - b ** L * torch.div(vis, b ** L, rounding_mode="floor")
    sel = b * lc[..., L - 1].long() + tail[:, None]
    return {"mean_kept_per_level": [round(float(v), 3) for v in lc.double().mean(dim=(0, 1))],
            "mean_selected_fraction": float((sel.double() / vis.double()[:, None]).mean())}


def decode_step_bytes(cand_rows: int, kept_nodes: int, b: int, tail: int, units: int,
                      queries: int, row: int):
    """Algorithmic bytes of one decode step, counted once per unit (a sequence
    and KV head, whose query heads share every read), with rows of `row` bytes:
    - selection: the distinct summary rows scored, the kept level-1 node list
      written (4 bytes per node) and the query rows read;
    - attention: the K and V rows of the kept nodes' tokens, the causal tail
      and token 0, the kept node list read back, the query rows read and the
      output rows written.
    Token 0 is counted once per unit even when its node is kept, at most one
    row over per unit. Returns (selection bytes, attention bytes, K/V rows)."""
    kv_rows = kept_nodes * b + units * (1 + tail)
    sel = cand_rows * row + kept_nodes * 4 + queries * row
    att = kv_rows * 2 * row + kept_nodes * 4 + 2 * queries * row
    return sel, att, kv_rows


def selection_per_query(lc, b: int, L: int, n: int, row: int) -> dict:
    """Per-query selection figures from kept counts lc [B][Hq][L] (top level
    first) of decode queries at position n - 1, with summary and K/V rows of
    `row` bytes:
    - the mean kept nodes per level and the mean fraction of the n visible
      tokens selected. A query selects b tokens per kept level-1 node, the
      tail past the last complete top node, and token 0 when node (1, 0) is
      not kept, so the fraction is exact to within one token per query;
    - the bytes the queries would touch if every query head read its own
      summary rows (the top nodes, then b per node kept above level 1), its
      own K and V rows and its index list: the sum over query heads, which
      counts the GQA duplication that the shared reads avoid."""
    top = n // b ** L
    tail = n - b ** L * top
    k = lc.long()
    sel = b * k[..., L - 1] + tail
    scored = top + b * k[..., :L - 1].sum(-1)
    return {"mean_kept_per_level": [round(float(v), 3) for v in lc.double().mean(dim=(0, 1))],
            "mean_selected_fraction": float((sel.double() / n).mean()),
            "bytes_per_q_head_sum": int((scored * row + sel * (2 * row + 8)).sum())}


def kernel_source_hash() -> str:
    """Hash of the decode-step kernels' code, comments and layout excluded, so
    that recorded DRAM counters stay tied to the code they were taken on."""
    h = hashlib.sha256()
    for f in ("decode_dense.cu", "attend.cu", "zha_device.cuh"):
        with open(os.path.join(ROOT, "tree_indexed_sparse_zha_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(strip_c_comments(fh.read()).encode())
            h.update(b"\0")
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "decode-deep-256k-b8_traffic.txt")
    try:
        vals = {}
        with open(path) as f:
            for ln in f:
                if ":" in ln and not ln.startswith("#"):
                    k, v = ln.split(":", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("kernel_source_hash") != kernel_source_hash():
            return None
        return vals
    except OSError:
        return None


# ---------------------------------------------------------------------------
# oracle CPU baseline (rank 0, bounded sample)
# ---------------------------------------------------------------------------

def oracle_rate(wl, n_queries: int, budget_s: float = 20.0):
    """Times the CPU oracle (tree for one (sequence, KV head) built untimed, then
    select + fp64 attention per query) on decode steps of that unit. Returns
    (queries/s, queries, seconds, queries flagged near-tie)."""
    import numpy as np

    import oracle

    c = wl.cfg
    K = wl.K[0, 0].float().cpu().numpy()
    V = wl.V[0, 0].float().cpu().numpy()
    R = wl.R.float().cpu().numpy()
    tr = oracle.build_tree(K, c.n_tokens, R, c.block, c.levels, True, c.capacity)
    done = flagged = 0
    t0 = time.perf_counter()
    step = 1
    while done < n_queries and time.perf_counter() - t0 < budget_s:
        q = wl.queries(step)[0].float().cpu().numpy()
        t = c.n_tokens + step - 1
        for h in range(c.group):
            idx, _, _, tie = oracle.select(q[h], tr, t, c.p)
            oracle.attend(q[h], K, V, idx)
            flagged += tie
            done += 1
            if done >= n_queries:
                break
        step += 1
    el = time.perf_counter() - t0
    return done / el, done, el, flagged


def oracle_prefill_rate(wl, n_queries: int, budget_s: float = 20.0):
    """Times the CPU oracle on chunk queries of KV head 0 (tree over the cached
    context and the chunk built untimed; select + fp64 attention per query).
    Returns (queries/s, queries, seconds, queries flagged near-tie)."""
    import numpy as np  # noqa: F401

    import oracle

    c = wl.cfg
    n = c.n_tokens + c.chunk
    K = wl.K[0, 0].float().cpu().numpy()
    V = wl.V[0, 0].float().cpu().numpy()
    R = wl.R.float().cpu().numpy()
    tr = oracle.build_tree(K, n, R, c.block, c.levels, True, c.capacity)
    q = wl.queries(0).float().cpu().numpy()
    done = flagged = 0
    t0 = time.perf_counter()
    i = 0
    while done < n_queries and time.perf_counter() - t0 < budget_s and i < c.chunk:
        for h in range(c.group):
            idx, _, _, tie = oracle.select(q[i, h], tr, c.n_tokens + i, c.p)
            oracle.attend(q[i, h], K, V, idx)
            flagged += tie
            done += 1
            if done >= n_queries:
                break
        i += 1
    el = time.perf_counter() - t0
    return done / el, done, el, flagged


def host_cpu():
    """(usable host cores, CPU model name)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return max(1, cores), model


def _widen_bf16(raw):
    import numpy as np

    return (raw.view(np.uint16).astype(np.uint32) << 16).view(np.float32)


def _oracle_worker(shm_name, shape, R, n_tree, b, L, cap, p, warm, steps, barrier, out_q):
    """One host core: rebuilds the unit's tree with the oracle and runs its
    warm-up steps (untimed), waits for every worker, then runs select + fp64
    attention over its timed steps."""
    import numpy as np
    from multiprocessing import shared_memory

    import oracle

    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        n = int(np.prod(shape))
        raw = np.ndarray((2 * n,), dtype=np.int16, buffer=shm.buf)
        K = _widen_bf16(raw[:n].copy()).reshape(shape)
        V = _widen_bf16(raw[n:].copy()).reshape(shape)
    finally:
        shm.close()
    tr = oracle.build_tree(K, n_tree, R, b, L, True, cap)
    for step in warm:
        for q, t in step:
            oracle.attend(q, K, V, oracle.select(q, tr, t, p)[0])
    barrier.wait()
    t0 = time.perf_counter()
    done = flagged = 0
    for step in steps:
        for q, t in step:
            idx, _, _, tie = oracle.select(q, tr, t, p)
            oracle.attend(q, K, V, idx)
            done += 1
            flagged += tie
    out_q.put((done, time.perf_counter() - t0, flagged))


def oracle_steps_parallel(wl, steps, n_tree, workers, warm=()):
    """Times the CPU oracle over `steps` (each a list of (q fp32[d], t)
    queries of sequence 0 / KV head 0) on `workers` host processes at once,
    steps dealt round-robin. A harness around the oracle, not oracle code:
    each worker rebuilds the unit's tree untimed, then all start together.
    Returns (queries done, wall seconds of the timed part, queries flagged
    near-tie)."""
    import multiprocessing as mp
    from multiprocessing import shared_memory

    c = wl.cfg
    K = wl.K[0, 0].cpu().contiguous().view(torch.int16).numpy()
    V = wl.V[0, 0].cpu().contiguous().view(torch.int16).numpy()
    R = wl.R.float().cpu().numpy()
    shm = shared_memory.SharedMemory(create=True, size=K.nbytes + V.nbytes)
    procs = []
    try:
        buf = memoryview(shm.buf)
        buf[:K.nbytes] = K.tobytes()
        buf[K.nbytes:K.nbytes + V.nbytes] = V.tobytes()
        del buf
        ctx = mp.get_context("spawn")  # never fork a process holding a CUDA context
        barrier = ctx.Barrier(workers + 1)
        out_q = ctx.Queue()
        for w in range(workers):
            pr = ctx.Process(target=_oracle_worker,
                             args=(shm.name, K.shape, R, n_tree, c.block, c.levels, c.capacity,
                                   c.p, list(warm[w::workers]), steps[w::workers], barrier,
                                   out_q))
            pr.start()
            procs.append(pr)
        barrier.wait(timeout=900)
        t0 = time.perf_counter()
        res = [out_q.get(timeout=1800) for _ in range(workers)]
        el = time.perf_counter() - t0
        for pr in procs:
            pr.join(timeout=60)
    finally:
        for pr in procs:
            if pr.is_alive():
                pr.kill()
        shm.close()
        shm.unlink()
    return sum(r[0] for r in res), el, sum(r[2] for r in res)


def decode_oracle_steps(wl, n_steps):
    """Reference-arm steps of the decode workload: step s is the G query heads
    of sequence 0 / KV head 0 at decode step s (one sixteenth of a workload
    step's queries)."""
    c = wl.cfg
    out = []
    for s in range(1, n_steps + 1):
        q = wl.queries(((s - 1) % max(c.steps, 1)) + 1)[0].float().cpu().numpy()
        t = c.n_tokens + ((s - 1) % max(c.steps, 1))
        out.append([(q[h], t) for h in range(c.group)])
    return out


def prefill_oracle_steps(wl, n_steps):
    """Reference-arm steps of the prefill workload: step i is the G query heads
    of KV head 0 for chunk token i."""
    c = wl.cfg
    q = wl.queries(0).float().cpu().numpy()
    return [[(q[i % c.chunk, h], c.n_tokens + i % c.chunk) for h in range(c.group)]
            for i in range(n_steps)]


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over the ranks of the default process group (x
    itself without one). Only this scalar crosses ranks: the replicas share no
    data."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(queries_per_step: int, steps: int, world: int, ms_total_max: float) -> float:
    """Whole-job queries/s: every rank runs `steps` steps of its own replica;
    the job takes as long as the slowest rank."""
    return queries_per_step * steps * world / (ms_total_max / 1e3)


L2_BYTES = 126e6


def l2_note(kv_gb: float) -> str:
    if kv_gb * 1e9 > L2_BYTES:
        return f"inputs larger than L2 (K+V {kv_gb:.2f} GB), no flush"
    return f"inputs fit in L2 (K+V {kv_gb:.3f} GB): a small diagnostic case, not a bench number"


def workload_config(args, c):
    if is_prefill(args.workload):
        kv_gb = 2 * c.n_kv_heads * c.capacity * c.head_dim * 2 / 1e9
        return {"workload": args.workload, "batch": c.batch, "context": c.n_tokens,
                "chunk": c.chunk, "heads": f"{c.n_q_heads}q/{c.n_kv_heads}kv",
                "head_dim": c.head_dim, "tree": f"b={c.block},L={c.levels}", "p": c.p,
                "queries_per_step": c.chunk * c.n_q_heads, "l2": l2_note(kv_gb)}
    kv_gb = 2 * c.batch * c.n_kv_heads * c.n_tokens * c.head_dim * (2 if c.dtype == "bf16" else 4) / 1e9
    return {"workload": args.workload, "batch": c.batch, "context": c.n_tokens,
            "heads": f"{c.n_q_heads}q/{c.n_kv_heads}kv", "head_dim": c.head_dim,
            "tree": f"b={c.block},L={c.levels}", "p": c.p,
            "queries_per_step": c.batch * c.n_q_heads, "l2": l2_note(kv_gb)}


def tree_build_work(n_tokens: int, b: int, L: int, D: int, units: int, elem: int = 2):
    """Algorithmic work of building every complete node over n_tokens tokens of
    `units` (sequence, KV head) units: (bytes, flops). Bytes: the keys read,
    every summary row read as a child of the level above, every summary row
    written. Flops: per child of a node, 16 reference-query dot products of
    length D and its share of the weighted sum (D), two flops per FMA."""
    rows = [units * (n_tokens // b ** l) for l in range(1, L + 1)]
    children = units * n_tokens + sum(rows[:-1])  # inputs of levels 1..L
    nbytes = (units * n_tokens + sum(rows[:-1]) + sum(rows)) * D * elem
    flops = 2.0 * (16 * D + D) * children
    return nbytes, flops


def fp32_peak_tflops(dev) -> float:
    """FP32 FMA peak of the device at its top SM clock: SMs x 128 lanes x 2 flops."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return sms * 128 * 2 * 1.965e9 / 1e12


def time_tree_build(cfg, cache, stream, reps: int = 3) -> float:
    import tree_indexed_sparse_zha_b200 as z

    z.zha_build_tree(cfg, cache)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    e0.record(stream)
    for _ in range(reps):
        z.zha_build_tree(cfg, cache)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def tree_builds_other_workloads(dev, peak_gbs: float) -> dict:
    """Tree-build rate of the other workloads' caches (the 32K decode, the wide
    256K tree and the 1M-token prefill context), built from scratch."""
    import tree_indexed_sparse_zha_b200 as z
    from tree_indexed_sparse_zha_b200 import workloads as W

    out = {}
    stream = torch.cuda.current_stream()
    for name in ("decode-deep-32k", "decode-wide-256k-b8", "prefill-deep-1m-chunk4k"):
        wl = W.make(name, device=dev, steps=0, chunk=0)
        c = wl.cfg
        cfg = z.make_config(c.head_dim, c.block, c.levels, c.n_q_heads, c.n_kv_heads, c.batch,
                            c.capacity, c.torch_dtype)
        cache = z.Cache(wl.K, wl.V, wl.R.float().contiguous(), z.alloc_tree(cfg, dev),
                        wl.seq_len.clone())
        ms = time_tree_build(cfg, cache, stream)
        nbytes, flops = tree_build_work(c.n_tokens, c.block, c.levels, c.head_dim,
                                        c.batch * c.n_kv_heads)
        out[name] = {"ms": ms, "tokens": c.batch * c.n_kv_heads * c.n_tokens,
                     "gb_per_s": nbytes / (ms / 1e3) / 1e9,
                     "hbm_frac": nbytes / (ms / 1e3) / 1e9 / peak_gbs,
                     "tflops": flops / (ms / 1e3) / 1e12,
                     "fp32_frac": flops / (ms / 1e3) / 1e12 / fp32_peak_tflops(dev)}
        del wl, cache
        torch.cuda.empty_cache()
    return out


def fp4_router_leg(z, cfg, cache, c, ws, st, queries, peak: float, steps: int = 20,
                   warmup: int = 3) -> dict:
    """The FP4 router variant on the headline cache as it stands (tree and
    lengths of the last timed step): the 4-bit copy's quantization time, then
    zha_decode_fp4 against zha_decode on the same queries (eager, no extend),
    the bytes each touches, and the drift of the variant's attended sets from
    the canonical ones (recall of the canonical set, size ratio), per
    (sequence, query head) of the last query set."""
    dev = queries.device
    B, Hq, Hkv, D, b, L = c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim, c.block, c.levels
    fp4 = z.alloc_fp4_tree(cfg, dev)
    z.zha_fp4_quantize_tree(cfg, cache, fp4)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    e0.record()
    z.zha_fp4_quantize_tree(cfg, cache, fp4)
    e1.record()
    torch.cuda.synchronize()
    quant_ms = e0.elapsed_time(e1)
    out = torch.empty_like(queries[0])
    n_q = queries.shape[0]

    def timed(fn):
        for i in range(warmup):
            fn(queries[i % n_q])
        torch.cuda.synchronize()
        e0.record()
        for i in range(steps):
            fn(queries[i % n_q])
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    canon_ms = timed(lambda q: z.zha_decode(cfg, cache, q, c.p, out, None, ws, st))
    fp4_ms = timed(lambda q: z.zha_decode_fp4(cfg, cache, fp4, q, c.p, out, None, ws, st))
    n = int(cache.seq_len.max().item())
    tail = n - b ** L * (n // b ** L)
    row = D * 2
    lists = {}
    bytes_ = {}
    for name, fn in (("canonical", lambda q: z.zha_decode(cfg, cache, q, c.p, out, None, ws, st)),
                     ("fp4", lambda q: z.zha_decode_fp4(cfg, cache, fp4, q, c.p, out, None, ws,
                                                        st))):
        fn(queries[(steps - 1) % n_q])
        stats = torch.zeros(B * Hkv, L + 1, dtype=torch.int32, device=dev)
        z.zha_decode_stats(cfg, ws, stats)
        idx = torch.empty(B, Hq, n + 2, dtype=torch.int32, device=dev)
        n_idx = torch.zeros(B, Hq, dtype=torch.int32, device=dev)
        z.zha_decode_kept_lists(cfg, cache, ws, idx, n_idx, st)
        torch.cuda.synchronize()
        stats = stats.cpu()
        cand, kept = int(stats[:, :L].sum()), int(stats[:, L].sum())
        srow = row if name == "canonical" else D // 2 + 2 * (D // 32)
        sel, att, _ = decode_step_bytes(cand, kept, b, tail, B * Hkv, B * Hq, row)
        sel += cand * (srow - row)
        bytes_[name] = (sel, att)
        lists[name] = (idx, n_idx.cpu())
    if int(st.item()) != 0:
        raise RuntimeError(f"fp4 leg: device status {z.status_string(int(st.item()))}")
    recall, ratio = [], []
    (ci, cn), (fi, fn_) = lists["canonical"], lists["fp4"]
    for s in range(B):
        for h in range(Hq):
            a = ci[s, h, :int(cn[s, h])]
            f = fi[s, h, :int(fn_[s, h])]
            recall.append(torch.isin(a, f).sum().item() / a.numel())
            ratio.append(f.numel() / a.numel())
    sel4, att4 = bytes_["fp4"]
    selc, attc = bytes_["canonical"]
    return {
        "format": "e2m1 codes, one int16 power-of-two exponent per 32 elements (72 B per "
                  "d=128 row instead of 256 B)",
        "quantize_ms": quant_ms,
        "decode_ms": {"fp4": fp4_ms, "canonical": canon_ms},
        "queries_per_s": {"fp4": B * Hq / (fp4_ms / 1e3), "canonical": B * Hq / (canon_ms / 1e3)},
        "select_bytes_per_step": {"fp4": sel4, "canonical": selc},
        "bytes_per_step": {"fp4": sel4 + att4, "canonical": selc + attc},
        "hbm_frac": {"fp4": (sel4 + att4) / (fp4_ms / 1e3) / 1e9 / peak,
                     "canonical": (selc + attc) / (canon_ms / 1e3) / 1e9 / peak},
        "recall_of_canonical_set": {"mean": sum(recall) / len(recall), "min": min(recall)},
        "set_size_ratio_mean": sum(ratio) / len(ratio),
    }


def wide_p_sweep(dev, peak: float, steps: int = 20, warmup: int = 3) -> list:
    """The wide-tree 256K workload (b = 256, one level, 8 sequences): decode
    steps (select + attend) at every p of its sweep, queries/s and the HBM
    fraction of the bytes each step touches."""
    import tree_indexed_sparse_zha_b200 as z
    from tree_indexed_sparse_zha_b200 import workloads as W

    wl = W.make("decode-wide-256k-b8", device=dev)
    c = wl.cfg
    cfg = z.make_config(c.head_dim, c.block, c.levels, c.n_q_heads, c.n_kv_heads, c.batch,
                        c.capacity, c.torch_dtype)
    cache = z.Cache(wl.K, wl.V, wl.R.float().contiguous(), z.alloc_tree(cfg, dev),
                    wl.seq_len.clone())
    z.zha_build_tree(cfg, cache)
    ws = z.alloc_workspace(cfg, z.ZHA_OP_DECODE, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    q = wl.queries(0)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    B, Hq, Hkv, D, b, L = c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim, c.block, c.levels
    n = c.n_tokens
    res = []
    for p in c.p_sweep:
        for _ in range(warmup):
            z.zha_decode(cfg, cache, q, p, out, None, ws, st)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            z.zha_decode(cfg, cache, q, p, out, None, ws, st)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        # kept counts per query: one more step on the same inputs, untimed
        lc = torch.zeros(B, Hq, L, dtype=torch.int32, device=dev)
        z.zha_decode(cfg, cache, q, p, out, lc, ws, st)
        stats = torch.zeros(B * Hkv, L + 1, dtype=torch.int32, device=dev)
        z.zha_decode_stats(cfg, ws, stats)
        stats = stats.cpu()
        top = n // b ** L
        sel_b, att_b, kv_rows = decode_step_bytes(int(stats[:, :L].sum()), int(stats[:, L].sum()),
                                                  b, n - b ** L * top, B * Hkv, B * Hq, D * 2)
        res.append({"p": p, "ms_per_step": ms, "queries_per_s": B * Hq / (ms / 1e3),
                    "bytes_touched_per_step": sel_b + att_b,
                    "kv_fraction_read": kv_rows / (B * Hkv * n),
                    "hbm_frac": (sel_b + att_b) / (ms / 1e3) / 1e9 / peak,
                    **selection_per_query(lc.cpu(), b, L, n, D * 2)})
    if int(st.item()) != 0:
        raise RuntimeError(f"wide sweep: device status {z.status_string(int(st.item()))}")
    del cache, ws, wl
    torch.cuda.empty_cache()
    return res


def prefill_chunk_leg(rank, world, dev, steps: int = 3, warmup: int = 3) -> dict:
    """The chunked-prefill workload at full size, timed as `--workload
    prefill-deep-1m-chunk4k` times it but over a few steps: one step is
    zha_prefill_chunk over the 4096-token chunk after 1,048,576 cached tokens.
    A failure is reported in the returned entry instead of ending the run."""
    a = argparse.Namespace(workload="prefill-deep-1m-chunk4k", steps=steps, warmup=warmup,
                           n_tokens=None)
    try:
        r, wl = run_prefill(a, rank, world, dev)
    except Exception as e:  # noqa: BLE001 -- recorded in the JSON line
        return {"error": f"{type(e).__name__}: {e}"[:300]}
    del wl
    torch.cuda.empty_cache()
    keep = ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "config", "selection",
            "tensor_core_top_level", "roofline", "tree_build", "e2e", "gpu_launches", "clocks")
    return {k: r[k] for k in keep}


def run_zha(args, rank, world, dev):
    import tree_indexed_sparse_zha_b200 as z
    from tree_indexed_sparse_zha_b200 import workloads as W

    z.lib()  # fail loudly if the extension is missing
    wl = W.make(args.workload, device=dev, n_tokens=args.n_tokens)
    c = wl.cfg
    n_steps_cap = c.steps
    cfg = z.make_config(c.head_dim, c.block, c.levels, c.n_q_heads, c.n_kv_heads, c.batch,
                        c.capacity, c.torch_dtype)
    B, Hq, Hkv, D, b, L = c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim, c.block, c.levels
    # per-step lengths and queries are precomputed inputs (resident in HBM)
    lens = (c.n_tokens + torch.arange(n_steps_cap + 1, device=dev, dtype=torch.int32))
    lens = lens.view(-1, 1).expand(-1, B).contiguous()           # [step][B]
    queries = torch.stack([wl.queries(s) for s in range(1, n_steps_cap + 1)])  # [step][B][Hq][D]
    tree = z.alloc_tree(cfg, dev)
    cache = z.Cache(wl.K, wl.V, wl.R.float().contiguous(), tree, lens[0])
    ws = z.alloc_workspace(cfg, z.ZHA_OP_DECODE, device=dev)
    wsd = z.alloc_workspace(cfg, z.ZHA_OP_DENSE, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, D, dtype=c.torch_dtype, device=dev)
    stream = torch.cuda.current_stream()

    # ---- tree build (rate reported; not part of a decode step) ----
    build_ms = time_tree_build(cfg, cache, stream)
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    n_tok = B * Hkv * c.n_tokens
    build_bytes, build_flops = tree_build_work(c.n_tokens, b, L, D, B * Hkv)

    def step_inputs(i):
        s = (i % n_steps_cap) + 1  # wrap: rebuilt nodes are identical
        return s, lens[s - 1], lens[s], queries[s - 1]

    # The timed step is one CUDA graph of zha_extend_tree + zha_decode (the
    # decode's unit groups on the library's own streams, joined back), fed
    # through static buffers: each step copies its lengths and queries into
    # them (inside the timed region) and replays the graph.
    old_st, len_st = lens[0].clone(), lens[0].clone()
    q_st = torch.empty_like(queries[0])
    cache.seq_len = len_st

    def load_inputs(i):
        _, old, new, q = step_inputs(i)
        old_st.copy_(old)
        len_st.copy_(new)
        q_st.copy_(q)

    def decode_body():
        z.zha_extend_tree(cfg, cache, old_st, 1)
        z.zha_decode(cfg, cache, q_st, c.p, out, None, ws, st)

    # reset the tree to the initial length, then warm up (eagerly, which also
    # creates the library's streams), capture and warm up the graph
    len_st.copy_(lens[0])
    z.zha_build_tree(cfg, cache)
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for i in range(args.warmup):
            load_inputs(i)
            decode_body()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    load_inputs(args.warmup)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        decode_body()
    torch.cuda.synchronize()
    len_st.copy_(lens[0])
    z.zha_build_tree(cfg, cache)
    for i in range(args.warmup):
        load_inputs(i)
        graph.replay()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {z.status_string(int(st.item()))}")

    t_start, t_end = torch.cuda.Event(True), torch.cuda.Event(True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for i in range(args.steps):
        load_inputs(args.warmup + i)
        graph.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_total = t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_total, dev)
    n_after = args.warmup + args.steps  # steps appended so far (for the phase loop below)
    ms_step = ms_total / args.steps
    queries_per_step = B * Hq
    value = throughput(queries_per_step, args.steps, world, ms_total)

    # ---- bytes touched per step (work counters of the last timed step) ----
    stats = torch.zeros(B * Hkv, L + 1, dtype=torch.int32, device=dev)
    z.zha_decode_stats(cfg, ws, stats)
    torch.cuda.synchronize()
    stats = stats.cpu()
    s_last, _, new_last, _ = step_inputs(args.warmup + args.steps - 1)
    n_last = int(new_last[0].item())
    top = n_last // b ** L
    tail = n_last - b ** L * top
    row = D * 2
    cand_rows = int(stats[:, :L].sum())
    kept_nodes = int(stats[:, L].sum())
    sel_bytes, att_bytes, kv_rows = decode_step_bytes(cand_rows, kept_nodes, b, tail, B * Hkv,
                                                      queries_per_step, row)
    # per-query kept counts of the last step's queries: one more select, untimed
    lc = torch.zeros(B, Hq, L, dtype=torch.int32, device=dev)
    z.zha_decode_select(cfg, cache, step_inputs(args.warmup + args.steps - 1)[3], c.p, lc, ws, st)
    torch.cuda.synchronize()
    per_query = selection_per_query(lc.cpu(), b, L, n_last, D * 2)

    # ---- phase split: the same steps eagerly on one stream, select and attend
    # apart (the roofline of each kernel group; not the headline) ----
    nph = min(20, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nph)]
    for i in range(nph):
        load_inputs(n_after + i)
        ev = evs[i]
        ev[0].record(stream)
        z.zha_extend_tree(cfg, cache, old_st, 1)
        ev[1].record(stream)
        z.zha_decode_select(cfg, cache, q_st, c.p, None, ws, st)
        ev[2].record(stream)
        z.zha_decode_attend(cfg, cache, q_st, out, ws)
        ev[3].record(stream)
    torch.cuda.synchronize()
    ms_ext, ms_sel, ms_att = (sum(e[a].elapsed_time(e[a + 1]) for e in evs) / nph
                              for a in range(3))
    ext_bytes = 0
    step_bytes = sel_bytes + att_bytes + ext_bytes
    peak, peak_kind = measured_peaks()
    hbm_frac = step_bytes / (ms_step / 1e3) / 1e9 / peak

    # ---- dense flash-decoding from the same library, same step inputs ----
    nd = min(20, args.steps)
    z.zha_dense_decode(cfg, cache, queries[0], out, wsd)
    torch.cuda.synchronize()
    e0.record()
    for i in range(nd):
        z.zha_dense_decode(cfg, cache, queries[i % n_steps_cap], out, wsd)
    e1.record()
    torch.cuda.synchronize()
    dense_ms = max_over_ranks(e0.elapsed_time(e1) / nd, dev)
    dense_bytes = B * Hkv * n_last * 2 * row + 2 * queries_per_step * row

    # ---- end to end through the API with host buffers ----
    ne = min(50, args.steps)
    kv_host = torch.empty(ne, 2, B, Hkv, D, dtype=c.torch_dtype).pin_memory()
    q_host = torch.empty(ne, B, Hq, D, dtype=c.torch_dtype).pin_memory()
    for i in range(ne):
        s, _, _, q = step_inputs(i)
        kv_host[i, 0].copy_(wl.K[:, :, c.n_tokens + s - 1])
        kv_host[i, 1].copy_(wl.V[:, :, c.n_tokens + s - 1])
        q_host[i].copy_(q)
    out_host = torch.empty(ne, B, Hq, D, dtype=c.torch_dtype).pin_memory()
    kv_dev = torch.empty(2, B, Hkv, D, dtype=c.torch_dtype, device=dev)
    q_dev = torch.empty(B, Hq, D, dtype=c.torch_dtype, device=dev)
    cache.seq_len = lens[0]
    z.zha_build_tree(cfg, cache)
    torch.cuda.synchronize()
    e0.record()
    for i in range(ne):
        s, old, new, _ = step_inputs(i)
        kv_dev.copy_(kv_host[i], non_blocking=True)
        q_dev.copy_(q_host[i], non_blocking=True)
        wl.K[:, :, c.n_tokens + s - 1] = kv_dev[0]
        wl.V[:, :, c.n_tokens + s - 1] = kv_dev[1]
        cache.seq_len = new
        z.zha_extend_tree(cfg, cache, old, 1)
        z.zha_decode(cfg, cache, q_dev, c.p, out, None, ws, st)
        out_host[i].copy_(out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / ne
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h2d = kv_host[0].numel() * kv_host.element_size() + q_host[0].numel() * q_host.element_size()
    d2h = out_host[0].numel() * out_host.element_size()

    # ---- roofline of both kernel groups; the line's `roofline` is the one
    # that takes longer. Traffic is ncu's DRAM bytes per launch from the
    # committed record, while it matches these kernels' sources ----
    traffic = recorded_traffic() if args.n_tokens is None else None  # taken at full size
    roof_att = {"kernel": "attend_mma_kernel + combine_kernel (zha_decode_attend)",
                "bound": "hbm", "achieved": att_bytes / (ms_att / 1e3) / 1e9, "peak": peak,
                "unit": "GB/s", "peak_kind": peak_kind,
                "traffic": float(traffic["attend_dram_bytes_per_step"]) if traffic else None}
    roof_sel = {"kernel": "dense_score_kernel + head_cut_kernel + union_kernel "
                          "(zha_decode_select)",
                "bound": "hbm", "achieved": sel_bytes / (ms_sel / 1e3) / 1e9, "peak": peak,
                "unit": "GB/s", "peak_kind": peak_kind,
                "traffic": float(traffic["select_dram_bytes_per_step"]) if traffic else None}
    for r_ in (roof_att, roof_sel):
        r_["frac"] = r_["achieved"] / r_["peak"]
    roof = dict(roof_att if ms_att >= ms_sel else roof_sel)

    res = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian-mixture keys, planted needles; no dataset)",
        "config": workload_config(args, c),
        "timed_step": "a CUDA graph of zha_extend_tree + zha_decode, replayed after the "
                      "step's lengths and queries are copied into its input buffers",
        "hbm_frac": hbm_frac,
        "hbm_frac_of_nominal_8tbs": step_bytes / (ms_step / 1e3) / 8e12,
        "bytes_touched_per_step": step_bytes,
        "phases_ms": {"extend": ms_ext, "select": ms_sel, "attend": ms_att},
        "selection": {"summary_rows_scored": cand_rows, "kept_level1_nodes": kept_nodes,
                      "kv_rows_read": kv_rows,
                      "kv_fraction_read": kv_rows / (B * Hkv * n_last), **per_query},
        "roofline": roof,
        "roofline_by_phase": {"select": roof_sel, "attend": roof_att},
        "dense": {"ms_per_step": dense_ms, "queries_per_s": queries_per_step * world / (dense_ms / 1e3),
                  "hbm_gbs": dense_bytes / (dense_ms / 1e3) / 1e9,
                  "hbm_frac": dense_bytes / (dense_ms / 1e3) / 1e9 / peak},
        "tree_build": {"ms": build_ms, "gb_per_s": build_bytes / (build_ms / 1e3) / 1e9,
                       "tflops": build_flops / (build_ms / 1e3) / 1e12,
                       "fp32_frac": build_flops / (build_ms / 1e3) / 1e12 / fp32_peak_tflops(dev),
                       "tokens": n_tok},
        "e2e": {"value": queries_per_step * world / (e2e_ms / 1e3), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        # per step: the extension, and per unit group (the library forms up to 4
        # groups of at least 2 (sequence, KV head) units) score, cut, union,
        # attention and combine
        "gpu_launches": (1 + 5 * min(4, max(1, B * Hkv // 2))) * args.steps,
        "clocks": clocks,
    }
    res["fp4_router"] = fp4_router_leg(z, cfg, cache, c, ws, st, queries, peak)
    if args.n_tokens is None:  # the other workloads at their full sizes
        res["decode_wide_p_sweep"] = wide_p_sweep(dev, peak)
        res["tree_build_other_workloads"] = tree_builds_other_workloads(dev, peak)
        res["prefill_chunk"] = prefill_chunk_leg(rank, world, dev)
    return res, wl


def run_prefill(args, rank, world, dev):
    """One step = zha_prefill_chunk over the whole chunk: the tree extended over
    the chunk, the top level of every (token, head) scored on the tensor cores
    and certified, the traversal and sparse attention for every query."""
    import tree_indexed_sparse_zha_b200 as z
    from tree_indexed_sparse_zha_b200 import workloads as W

    z.lib()  # fail loudly if the extension is missing
    wl = W.make(args.workload, device=dev, n_tokens=args.n_tokens)
    c = wl.cfg
    cfg = z.make_config(c.head_dim, c.block, c.levels, c.n_q_heads, c.n_kv_heads, c.batch,
                        c.capacity, c.torch_dtype)
    Hq, Hkv, D, b, L, T, G = (c.n_q_heads, c.n_kv_heads, c.head_dim, c.block, c.levels, c.chunk,
                              c.group)
    start = c.n_tokens
    len0 = torch.full((1,), start, dtype=torch.int32, device=dev)
    len1 = torch.full((1,), start + T, dtype=torch.int32, device=dev)
    cache = z.Cache(wl.K, wl.V, wl.R.float().contiguous(), z.alloc_tree(cfg, dev), len0)
    ws = z.alloc_workspace(cfg, z.ZHA_OP_PREFILL, T, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    q = wl.queries(0)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)

    # ---- tree over the cached context (rate reported; not part of a step) ----
    build_ms = time_tree_build(cfg, cache, stream)

    def one_step():
        cache.seq_len = len1
        z.zha_prefill_chunk(cfg, cache, q, 0, start, c.p, out, None, ws, st)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {z.status_string(int(st.item()))}")
    t_start, t_end = torch.cuda.Event(True), torch.cuda.Event(True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for _ in range(args.steps):
        one_step()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev)
    ms_step = ms_total / args.steps
    queries_per_step = T * Hq
    value = throughput(queries_per_step, args.steps, world, ms_total)

    # ---- kept counts per (token, head): one more step, untimed ----
    lc = torch.zeros(T, Hq, L, dtype=torch.int32, device=dev)
    cache.seq_len = len1
    z.zha_prefill_chunk(cfg, cache, q, 0, start, c.p, out, lc, ws, st)
    torch.cuda.synchronize()
    selection = prefill_selection(lc.cpu(), b, L, start)

    # ---- the tensor-core top level alone (GEMM + certificates) ----
    cert = torch.full((T, Hq), -1, dtype=torch.int32, device=dev)
    z.zha_prefill_top_scores(cfg, cache, q, 0, start, c.p, None, cert, ws, st)
    torch.cuda.synchronize()
    nr = 20
    e0.record(stream)
    for _ in range(nr):
        z.zha_prefill_top_scores(cfg, cache, q, 0, start, c.p, None, cert, ws, st)
    e1.record(stream)
    torch.cuda.synchronize()
    top_ms = max_over_ranks(e0.elapsed_time(e1) / nr, dev)
    n_top = min((start + T) // b ** L, c.capacity // b ** L)
    gemm_flops = 2.0 * T * Hq * n_top * D
    # algorithmic bytes: query rows, top summaries, the fp32 scores written by
    # the GEMM and read by the certifier, and the per-unit seeds
    top_bytes = (T * Hq * D * 2 + Hkv * n_top * D * 2 + 2 * T * Hq * n_top * 4
                 + T * Hkv * (n_top + 4 + 4 * G))
    cert_heads = float((cert == 1).float().mean())
    cert_units = float((cert == 1).view(T, Hkv, G).all(-1).float().mean())

    # ---- end to end with host buffers: the chunk's K/V rows and queries in,
    # the outputs back, every step ----
    ne = min(3, args.steps)
    kv_host = torch.stack([wl.K[0, :, start:start + T], wl.V[0, :, start:start + T]]).cpu()
    kv_host = kv_host.pin_memory()
    q_host = q.cpu().pin_memory()
    out_host = torch.empty_like(q_host).pin_memory()
    kv_dev = torch.empty_like(kv_host, device=dev)
    q_dev = torch.empty_like(q)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(ne):
        kv_dev.copy_(kv_host, non_blocking=True)
        q_dev.copy_(q_host, non_blocking=True)
        wl.K[0, :, start:start + T] = kv_dev[0]
        wl.V[0, :, start:start + T] = kv_dev[1]
        cache.seq_len = len1
        z.zha_prefill_chunk(cfg, cache, q_dev, 0, start, c.p, out, None, ws, st)
        out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / ne, dev)
    h2d = kv_host.numel() * kv_host.element_size() + q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {z.status_string(int(st.item()))}")

    peak, peak_kind = measured_peaks()
    roof = {"kernel": "tensor-core top level: top_score_tc_kernel + top_certify_kernel "
                      "(zha_prefill_top_scores)", "bound": "hbm",
            "achieved": top_bytes / (top_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
            "peak_kind": peak_kind, "traffic": None}
    roof["frac"] = roof["achieved"] / roof["peak"]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tile = max(1, min(T, (2 * sms) // Hkv))
    tiles = (T + tile - 1) // tile
    # fill, tree levels, top level (norms, GEMM, certificates), then per query
    # tile positions, traversal, attention and combine
    launches = 1 + L + 3 + 4 * tiles
    res = {
        "metric": PREFILL_METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian-mixture keys, planted needles; no dataset)",
        "config": workload_config(args, c),
        "selection": selection,
        "tensor_core_top_level": {
            "ms": top_ms, "top_nodes": n_top, "gemm_flops": gemm_flops,
            "gemm_tflops_incl_certify": gemm_flops / (top_ms / 1e3) / 1e12,
            "certified_head_fraction": cert_heads, "certified_unit_fraction": cert_units},
        "roofline": roof,
        "tree_build": {"ms": build_ms, "tokens": Hkv * start},
        "e2e": {"value": queries_per_step * world / (e2e_ms / 1e3), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
    }
    return res, wl


# tree geometries of the sweep: b^L in [256, 16384], at most 8 levels
SWEEP_GEOMETRIES = [(2, 8), (4, 4), (4, 5), (4, 6), (4, 7), (8, 3), (8, 4), (16, 2), (16, 3),
                    (64, 2), (256, 1)]


def run_sweep(args, dev):
    """Decode steps (select + attend, cache fixed) of the 256K B = 8 workload
    for each tree geometry, beside the dense kernel on the same cache."""
    import tree_indexed_sparse_zha_b200 as z
    from tree_indexed_sparse_zha_b200 import workloads as W

    z.lib()
    peak, peak_kind = measured_peaks()
    base = W.CONFIGS[WORKLOAD]
    n_tok = args.n_tokens or base.n_tokens
    wl = W.make(WORKLOAD, device=dev, n_tokens=n_tok, steps=0)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    steps = min(args.steps, 50)
    queries = [wl.queries(s) for s in range(1, steps + 1)]
    for b, L in SWEEP_GEOMETRIES:
        c = wl.cfg
        cfg = z.make_config(c.head_dim, b, L, c.n_q_heads, c.n_kv_heads, c.batch, c.capacity,
                            c.torch_dtype)
        cache = z.Cache(wl.K, wl.V, wl.R.float().contiguous(), z.alloc_tree(cfg, dev),
                        wl.seq_len.clone())
        z.zha_build_tree(cfg, cache)
        ws = z.alloc_workspace(cfg, z.ZHA_OP_DECODE, device=dev)
        wsd = z.alloc_workspace(cfg, z.ZHA_OP_DENSE, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        out = torch.empty_like(queries[0])
        for i in range(args.warmup):
            z.zha_decode(cfg, cache, queries[i % steps], c.p, out, None, ws, st)
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"b={b} L={L}: {z.status_string(int(st.item()))}")
        e0.record(stream)
        for i in range(steps):
            z.zha_decode(cfg, cache, queries[i], c.p, out, None, ws, st)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        stats = torch.zeros(c.batch * c.n_kv_heads, L + 1, dtype=torch.int32, device=dev)
        z.zha_decode_stats(cfg, ws, stats)
        z.zha_dense_decode(cfg, cache, queries[0], out, wsd)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(steps):
            z.zha_dense_decode(cfg, cache, queries[i], out, wsd)
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / steps
        stats = stats.cpu()
        units = c.batch * c.n_kv_heads
        row = c.head_dim * 2
        top = n_tok // b ** L
        tail = n_tok - b ** L * top
        kept = int(stats[:, L].sum())
        q = c.batch * c.n_q_heads
        sel_b, att_b, kv_rows = decode_step_bytes(int(stats[:, :L].sum()), kept, b, tail, units,
                                                  q, row)
        touched = sel_b + att_b
        line = {"sweep": WORKLOAD, "block": b, "levels": L, "top_span": b ** L,
                "context": n_tok, "p": c.p, "steps": steps,
                "ms_per_step": ms, "queries_per_s": q / (ms / 1e3),
                "dense_ms_per_step": dense_ms, "dense_queries_per_s": q / (dense_ms / 1e3),
                "kv_fraction_read": kv_rows / (units * n_tok),
                "summary_rows_scored": int(stats[:, :L].sum()),
                "bytes_touched_per_step": touched,
                "hbm_frac": touched / (ms / 1e3) / 1e9 / peak, "peak_kind": peak_kind}
        print(json.dumps(line), flush=True)
        del cache, ws, wsd
        torch.cuda.empty_cache()


def cpu_baseline(wl, prefill: bool) -> dict:
    """The oracle on the host: every usable core at once (a bounded sample,
    a few steps per process), beside one core as the oracle stands."""
    c = wl.cfg
    cores, model = host_cpu()
    workers = min(cores, 8 if prefill else 32)
    steps = (prefill_oracle_steps if prefill else decode_oracle_steps)(wl, 3 * workers)
    n_tree = c.n_tokens + c.chunk if prefill else c.n_tokens
    done, el, flagged = oracle_steps_parallel(wl, steps, n_tree, workers)
    if prefill:
        r1, d1, e1, f1 = oracle_prefill_rate(wl, 200, budget_s=15.0)
        what = "chunk queries of KV head 0"
    else:
        r1, d1, e1, f1 = oracle_rate(wl, 200, budget_s=15.0)
        what = "decode queries of sequence 0 / KV head 0"
    return {"value": done / el, "unit": "queries/s", "cores": workers, "cpu_model": model,
            "host_cores": cores, "kind": "oracle", "near_tie_flagged": flagged,
            "sample": f"{done} {what} on {workers} processes in {el:.1f} s (trees built "
                      "untimed)",
            "single_core": {"value": r1, "unit": "queries/s", "cores": 1,
                            "near_tie_flagged": f1,
                            "sample": f"{d1} {what} in {e1:.1f} s (tree built untimed)"}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        from tree_indexed_sparse_zha_b200 import workloads as W

        dev = "cuda" if torch.cuda.is_available() else "cpu"
        wl = W.make(args.workload, device=dev, n_tokens=args.n_tokens)
        c = wl.cfg
        cores, model = host_cpu()
        prefill = is_prefill(args.workload)
        # workers hold the unit's K/V in fp32 and its tree: about 0.6 GB each at
        # 256K context, 1.5 GB at 1M
        workers = min(cores, 8 if prefill else 32, max(args.steps, 1))
        make_steps = prefill_oracle_steps if prefill else decode_oracle_steps
        all_steps = make_steps(wl, args.warmup + args.steps)
        n_tree = c.n_tokens + c.chunk if prefill else c.n_tokens
        done, el, flagged = oracle_steps_parallel(wl, all_steps[args.warmup:], n_tree, workers,
                                                  warm=all_steps[:args.warmup])
        rate = done / el
        step_desc = (f"the {c.group} query heads of KV head 0 for one chunk token"
                     if prefill else
                     f"the {c.group} query heads of sequence 0 / KV head 0 at one decode step")
        frac = (f"1/{c.chunk * c.n_kv_heads} of a chunk's queries" if prefill
                else f"1/{c.batch * c.n_kv_heads} of a workload step's queries")
        line = {"impl": "reference", "metric": PREFILL_METRIC if prefill else METRIC,
                "value": rate, "unit": "queries/s", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
                "step": f"{step_desc} ({frac}); steps dealt over {workers} host processes",
                "queries_timed": done,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32 select / f64 attention", "data": "synthetic",
                "config": workload_config(args, c),
                "cpu_baseline": {"value": rate, "unit": "queries/s", "cores": workers,
                                 "cpu_model": model, "host_cores": cores, "kind": "oracle",
                                 "near_tie_flagged": flagged,
                                 "sample": f"{done} queries ({args.steps} steps of {step_desc}) "
                                           f"in {el:.1f} s on {workers} processes, trees built "
                                           "untimed"},
                "e2e": {"value": rate, "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    if args.sweep:
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        if rank == 0:
            run_sweep(args, dev)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    prefill = is_prefill(args.workload)
    res, wl = (run_prefill if prefill else run_zha)(args, rank, world, dev)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl, prefill)
        else:
            res["cpu_baseline"] = None
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
