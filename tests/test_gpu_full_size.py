"""The decode workloads at full size, in the launch configuration the bench
times, against the CPU oracle (run over all host cores, one task per
(sequence, KV head) unit).

Bar: per-level kept counts and the token set each query head attends
(zha_decode_kept_lists: the rows the decode attention reads) bit-exact;
attention outputs within max-abs 2e-2 of the oracle's fp64 attention over its
own selection; summary trees bitwise."""
import numpy as np
import pytest
import torch

import tree_indexed_sparse_zha_b200 as z
from tree_indexed_sparse_zha_b200 import workloads as W

from _harness import TOL, Gpu
from _oracle_pool import fingerprint, run_units, unit_tree_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _gpu_fingerprints(idx: torch.Tensor, n_idx: torch.Tensor, pairs):
    """fingerprint() of the device lists of the given (sequence, head) pairs."""
    out = {}
    for s, h in pairs:
        n = int(n_idx[s, h])
        out[(s, h)] = fingerprint(idx[s, h, :n].cpu().numpy())
    return out


def _unit_tasks(wl, units_queries, n_tree, want_tree=False, with_v=True):
    c = wl.cfg
    R = wl.R.float().cpu().numpy()
    tasks = []
    for (s, kvh), qs in sorted(units_queries.items()):
        tasks.append({"unit": (s, kvh), "k": wl.K[s, kvh].cpu(),
                      "v": wl.V[s, kvh].cpu() if with_v else None, "dtype": c.dtype, "R": R,
                      "n_tree": n_tree, "b": c.block, "L": c.levels, "cap": c.capacity,
                      "queries": qs, "want_tree": want_tree})
    return tasks


def _compare_tree_rows(gpu: Gpu, s: int, kvh: int, rows: np.ndarray):
    c = gpu.c
    exp = unit_tree_rows(rows, c.capacity, c.block, c.levels)
    got = gpu.tree_unit(s, kvh)
    for l in range(1, c.levels + 1):
        a, b = got[l - 1], exp[l - 1]
        n = min(a.shape[0], b.shape[0])
        assert np.array_equal(a[:n].view(np.uint32), b[:n].view(np.uint32)), \
            f"unit ({s}, {kvh}) level {l}: {int((a[:n] != b[:n]).any(1).sum())} rows differ"


def test_decode_deep_256k_full_incremental():
    """The headline run as the bench times it: 8 sequences of 262,144 tokens,
    256 steps of zha_extend_tree (one appended token per sequence) and
    zha_decode. Every query of steps 1, 2, 128 and 256 is checked in full
    (counts, attended set element by element, output); a seeded 2 % of the
    other steps' queries in full too; then the final tree of all 16 units
    bitwise and the dense kernel of the last step against the oracle's dense
    attention."""
    wl = W.make("decode-deep-256k-b8", device="cuda")
    c = wl.cfg
    gpu = Gpu(wl)
    G = c.group
    full_steps = (1, 2, 128, 256)
    rng = np.random.default_rng(20261202)
    sampled = {s: [divmod(int(x), c.n_q_heads) for x in
                   rng.choice(c.batch * c.n_q_heads, 3, replace=False)]
               for s in range(1, c.steps + 1) if s not in full_steps}
    ws = gpu.decode_ws()
    old = gpu.cache.seq_len.clone()
    got = {}      # (step, seq, head) -> (counts, fingerprint, list or None, output)
    queries = {}  # (seq, kvh) -> oracle queries
    for step in range(1, c.steps + 1):
        old.copy_(gpu.cache.seq_len)
        gpu.cache.seq_len.add_(1)
        z.zha_extend_tree(gpu.cfg, gpu.cache, old, 1)
        q = wl.queries(step).to(gpu.dev)
        out = torch.empty_like(q)
        lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
        z.zha_decode(gpu.cfg, gpu.cache, q, c.p, out, lc, ws, gpu.status)
        idx, n_idx = gpu.kept_lists(ws)
        pairs = ([(s, h) for s in range(c.batch) for h in range(c.n_q_heads)]
                 if step in full_steps else sampled[step])
        t = c.n_tokens + step - 1
        lcn, outn, nn = lc.cpu().numpy(), out.float().cpu().numpy(), n_idx.cpu().numpy()
        qf = q.float().cpu().numpy()
        fps = _gpu_fingerprints(idx, n_idx, pairs)
        for s, h in pairs:
            lst = idx[s, h, :nn[s, h]].cpu().numpy() if step in full_steps else None
            got[(step, s, h)] = (lcn[s, h], fps[(s, h)], lst, outn[s, h])
            queries.setdefault((s, h // G), []).append(((step, s, h), qf[s, h], t, c.p, "full"))
        del idx, n_idx
    gpu.check_status()
    # dense flash-decoding of the last step against the oracle's dense attention
    qd = wl.queries(c.steps).to(gpu.dev)
    dense = gpu.dense(qd)
    qdf = qd.float().cpu().numpy()
    t_last = c.n_tokens + c.steps - 1
    for s in (0, 7):
        for h in range(c.n_q_heads):
            queries[(s, h // G)].append((("dense", s, h), qdf[s, h], t_last, 1.0, "dense"))
    final_n = c.n_tokens + c.steps
    res = run_units(_unit_tasks(wl, queries, final_n, want_tree=True))
    checked = flagged = 0
    for (s, kvh), results, rows in res:
        _compare_tree_rows(gpu, s, kvh, rows)
        for r in results:
            key = r["key"]
            if key[0] == "dense":
                err = np.abs(dense[key[1], key[2]] - r["dense"]).max()
                assert err < TOL["bf16"], (key, err)
                continue
            counts, fp, lst, o = got[key]
            assert counts.tolist() == r["counts"].tolist(), (key, counts, r["counts"])
            assert fp == r["fp"], key
            if lst is not None:
                assert np.array_equal(lst, r["idx"]), key
            err = np.abs(o - r["out"]).max()
            assert err < TOL["bf16"], (key, err)
            checked += 1
            flagged += r["tie"]
    assert checked == 4 * c.batch * c.n_q_heads + 3 * (c.steps - 4)


def test_decode_wide_256k_full_p_sweep():
    """The wide-tree workload (b = 256, one level, 1024 top nodes) at full
    size: p in {0.8, 0.9, 0.95, 0.99, 1.0} on sequences 2 and 5 (all 16 heads),
    counts, attended sets and outputs against the oracle; at p = 1 every
    visible token is attended, and the dense kernel is checked against the
    oracle's dense attention."""
    wl = W.make("decode-wide-256k-b8", device="cuda")
    c = wl.cfg
    gpu = Gpu(wl)
    G = c.group
    seqs = (2, 5)
    q = wl.queries(0).to(gpu.dev)
    qf = q.float().cpu().numpy()
    t = c.n_tokens - 1
    got = {}
    queries = {}
    for p in c.p_sweep:
        out, lc, idx, n_idx = gpu.decode(q, p, lists=True)
        nn = n_idx.cpu().numpy()
        for s in seqs:
            for h in range(c.n_q_heads):
                lst = idx[s, h, :nn[s, h]].cpu().numpy()
                if p >= 1.0:
                    assert np.array_equal(lst, np.arange(t + 1)), (s, h)
                got[(p, s, h)] = (lc[s, h], lst, out[s, h])
                queries.setdefault((s, h // G), []).append(((p, s, h), qf[s, h], t, p, "full"))
        del idx, n_idx
    dense = gpu.dense(q)
    for s in seqs:
        for h in range(c.n_q_heads):
            queries[(s, h // G)].append((("dense", s, h), qf[s, h], t, 1.0, "dense"))
    res = run_units(_unit_tasks(wl, queries, c.n_tokens, want_tree=True))
    for (s, kvh), results, rows in res:
        _compare_tree_rows(gpu, s, kvh, rows)
        for r in results:
            key = r["key"]
            if key[0] == "dense":
                assert np.abs(dense[key[1], key[2]] - r["dense"]).max() < TOL["bf16"], key
                continue
            counts, lst, o = got[key]
            assert counts.tolist() == r["counts"].tolist(), key
            assert np.array_equal(lst, r["idx"]), key
            assert np.abs(o - r["out"]).max() < TOL["bf16"], key
