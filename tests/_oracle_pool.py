"""The CPU oracle over many queries on all host cores, for the GPU parity
tests of full-size workloads.

Worker processes are spawned, never forked: a process forked from one that
holds a CUDA context can hang. Each task covers one (sequence, KV head) unit:
the worker rebuilds that unit's tree with the oracle, then selects (and, on
request, attends) every query given for it. Nothing here computes any of the
method's arithmetic; it only moves arrays to and from ``oracle``.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

import oracle


def fingerprint(idx: np.ndarray) -> Tuple[int, int, int, int]:
    """(length, sum, sum of squares, position-weighted sum) of an ascending
    index list: equal lists give equal fingerprints, and two different
    ascending lists of token positions below 2^24 agree on all four only by
    coincidence. Exact in int64 for lists this long."""
    a = np.asarray(idx, dtype=np.int64)
    w = np.arange(1, a.shape[0] + 1, dtype=np.int64)
    return (int(a.shape[0]), int(a.sum()), int((a * a).sum()), int((a * w).sum()))


def _widen(raw: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":  # raw holds the bf16 bit patterns as int16
        return (raw.view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    return raw.view(np.float32)


def _unit_task(args):
    (unit, kraw, vraw, dtype, R, n_tree, b, L, cap, queries, want_tree) = args
    K = _widen(kraw, dtype)
    V = _widen(vraw, dtype) if vraw is not None else None
    tr = oracle.build_tree(K, n_tree, R, b, L, dtype == "bf16", cap)
    out = []
    for key, q, t, p, mode in queries:
        idx, counts, _, tie = oracle.select(q, tr, t, p)
        r = {"key": key, "counts": counts.copy(), "tie": bool(tie), "fp": fingerprint(idx)}
        if mode in ("list", "full"):
            r["idx"] = idx
        if mode == "full":
            r["out"] = oracle.attend(q, K, V, idx)
        if mode == "dense":
            r["dense"] = oracle.dense(q, K, V, t)
        out.append(r)
    return unit, out, (tr.rows if want_tree else None)


def host_cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def run_units(tasks: Sequence[dict], workers: Optional[int] = None) -> List:
    """tasks: dicts with keys unit (any label), k, v (CPU torch tensors
    [Ncap][d] of one (sequence, KV head), bf16 or fp32; v may be None), dtype,
    R, n_tree, b, L, cap, queries [(key, q fp32[d], t, p, mode)] with mode one
    of "counts", "list" (adds the index list), "full" (adds the list and the
    fp64 attention output), "dense" (adds the fp64 dense output over [0, t]),
    and want_tree. Several tasks may share a unit (each rebuilds its tree).
    Returns [(unit, results, tree rows or None)] in task order."""
    import torch

    def raw(x):
        if x is None:
            return None
        x = x.contiguous()
        return (x.view(torch.int16) if x.dtype == torch.bfloat16 else x.float()).numpy()

    args = [(t["unit"], raw(t["k"]), raw(t.get("v")), t["dtype"], np.asarray(t["R"], np.float32),
             t["n_tree"], t["b"], t["L"], t["cap"], t["queries"], t.get("want_tree", False))
            for t in tasks]
    n = min(workers or host_cores(), len(args))
    if n <= 1:
        res = [_unit_task(a) for a in args]
    else:
        with mp.get_context("spawn").Pool(n) as pool:
            res = pool.map(_unit_task, args, chunksize=1)
    return res


def unit_tree_rows(rows: np.ndarray, n_cap: int, b: int, L: int) -> List[np.ndarray]:
    """The oracle's packed rows of one unit split per level (1..L)."""
    offs, _ = oracle.level_row_offsets(n_cap, b, L)
    out = []
    for l in range(1, L + 1):
        s = int(offs[l - 1])
        e = int(offs[l]) if l < L else rows.shape[0]
        out.append(rows[s:e])
    return out
