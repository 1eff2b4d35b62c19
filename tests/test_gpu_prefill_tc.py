"""Prefill top level on the tensor cores (tcgen05 GEMM + certificate) vs the oracle.

zha_prefill_top_scores scores the top level of every (token, head) of a chunk
with one bf16 GEMM per KV head and certifies each row. Checked here:
- the tensor-core scores z~ stay within the accumulation error model the
  certificate is built on, against the exact (fp64) score of the same bf16
  operands, and within a quarter of the certificate's bound of the oracle's
  canonical fp32 score (the certificate's safety factor is 4);
- the certificate's claim itself: for a certified row the canonical cut taken
  on z~ equals the canonical cut taken on the oracle's scores (both vectors lie
  in the certified box);
- enough rows certify for the fast path to run;
- zha_prefill_chunk, which skips the top level of certified units, still
  matches the oracle (level counts bit-exact, outputs within tolerance)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tree_indexed_sparse_zha_b200 import workloads as W

from _harness import TOL, Gpu, Ref, compare_tree

pytestmark = pytest.mark.gpu

z = __import__("tree_indexed_sparse_zha_b200")


def _top_case(cfg):
    """Workload with its tree built over the chunk too (seq_len = start + chunk)."""
    wl = W.Workload(cfg)
    c = wl.cfg
    gpu = Gpu(wl, build=False)
    start = c.n_tokens
    gpu.cache.seq_len.fill_(start + c.chunk)
    z.zha_build_tree(gpu.cfg, gpu.cache)
    torch.cuda.synchronize()
    ref = Ref(wl, start + c.chunk)
    return wl, gpu, ref, start


def _top_scores(gpu, q, start, p):
    c = gpu.c
    cap = c.capacity // c.block ** c.levels
    zt = torch.full((c.chunk, c.n_q_heads, cap), float("nan"), dtype=torch.float32,
                    device=gpu.dev)
    cert = torch.full((c.chunk, c.n_q_heads), -1, dtype=torch.int32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, c.chunk, device=gpu.dev)
    z.zha_prefill_top_scores(gpu.cfg, gpu.cache, q, 0, start, p, zt, cert, ws, gpu.status)
    gpu.check_status()
    return zt.cpu().numpy(), cert.cpu().numpy(), cap


def _check_top_scores(wl, gpu, ref, start, sample_tokens, min_cert_frac):
    c = wl.cfg
    L, b, d = c.levels, c.block, c.head_dim
    q = wl.queries(0).to(gpu.dev)
    zt, cert, cap = _top_scores(gpu, q, start, c.p)
    assert set(np.unique(cert).tolist()) <= {0, 1}
    qf = q.float().cpu().numpy().astype(np.float64)
    inv = float(np.float32(1.0 / math.sqrt(d)))
    lns = float(np.float32(L * math.log(b)))
    n_top = np.minimum((start + np.arange(c.chunk) + 1) // b ** L, cap)
    worst = 0.0
    for kvh in range(c.n_kv_heads):
        S = ref.tree(0, kvh).level(L).astype(np.float64)  # [cap][d], bf16 values
        snorm = np.linalg.norm(S, axis=1)
        for h in range(kvh * c.group, (kvh + 1) * c.group):
            Q = qf[:, h]                                   # [chunk][d]
            exact = (Q @ S.T) * inv + lns                  # fp64 score of the same operands
            unit = d * 2.0 ** -24 * inv * np.linalg.norm(Q, axis=1)[:, None] * snorm[None, :]
            valid = np.arange(cap)[None, :] < n_top[:, None]
            got = zt[:, h].astype(np.float64)
            assert np.isfinite(got[valid]).all()
            err = np.abs(got - exact)
            # accumulation (two sums of d exact products, one of them truncating)
            # plus the two rounded epilogue operations
            model = 2.0 * unit + 2.0 ** -22 * (np.abs(got) + lns + 1.0)
            assert (err[valid] <= model[valid]).all(), float((err - model)[valid].max())
            worst = max(worst, float((err / (unit + 1e-300))[valid].max()))
    # the certificate's bound (safety factor 4) against the canonical fp32 score
    cut_checked = 0
    for i in sample_tokens:
        n = int(n_top[i])
        nodes = np.arange(n, dtype=np.int64)
        for h in range(c.n_q_heads):
            kvh = h // c.group
            S = ref.tree(0, kvh).level(L)
            zc = np.array([oracle.score(qf[i, h], S[j], L, b) for j in range(n)],
                          dtype=np.float64)
            got = zt[i, h, :n].astype(np.float64)
            qn = float(np.linalg.norm(qf[i, h]))
            sn = np.linalg.norm(S[:n].astype(np.float64), axis=1)
            delta = 12.0 * d * 2.0 ** -24 * inv * qn * sn + 2.0 ** -21 * (2 * np.abs(got) + lns + 1)
            assert (np.abs(got - zc) <= delta / 4).all(), (i, h)
            if cert[i, h] == 1:
                k_tc, _, _, _ = oracle.cut(got.astype(np.float32), nodes, c.p)
                k_can, _, _, _ = oracle.cut(zc.astype(np.float32), nodes, c.p)
                assert np.array_equal(k_tc, k_can), (i, h)
                cut_checked += 1
    frac = float((cert == 1).mean())
    assert frac >= min_cert_frac, frac
    assert cut_checked > 0
    print(f"certified {frac:.3f}; worst |z~ - z| / (d 2^-24 inv |q||s|) = {worst:.3f}")
    return frac


def test_top_scores_many_nodes():
    """515 top nodes (three N tiles, the last one ragged) and 2400 rows per KV
    head (a ragged M tile): b = 4, L = 3, a 300-token chunk after 32700 tokens."""
    base = W.CONFIGS["prefill-deep-1m-chunk4k"]
    wl, gpu, ref, start = _top_case(base.scaled(32700, chunk=300, levels=3))
    compare_tree(gpu, ref, 0, 0)
    compare_tree(gpu, ref, 0, 1)
    _check_top_scores(wl, gpu, ref, start, [0, 1, 150, 298, 299], 0.3)


def test_top_scores_chunk_crossing_node():
    """Deep tree (b = 4, L = 6): the chunk completes a top node midway, so the
    GEMM's N exceeds what the early tokens may see."""
    base = W.CONFIGS["prefill-deep-1m-chunk4k"]
    wl, gpu, ref, start = _top_case(base.scaled(16256, chunk=256))
    _check_top_scores(wl, gpu, ref, start, [0, 126, 127, 128, 255], 0.3)


def test_prefill_chunk_many_nodes_parity():
    """zha_prefill_chunk on the 515-node geometry: certified units start one
    level below the top, the rest score it canonically; both match the oracle."""
    base = W.CONFIGS["prefill-deep-1m-chunk4k"]
    wl = W.Workload(base.scaled(32700, chunk=300, levels=3))
    c = wl.cfg
    gpu = Gpu(wl)
    start = c.n_tokens
    gpu.cache.seq_len.fill_(start + c.chunk)
    q = wl.queries(0).to(gpu.dev)
    out = torch.empty_like(q)
    lc = torch.full((c.chunk, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, c.chunk, device=gpu.dev)
    z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out, lc, ws, gpu.status)
    gpu.check_status()
    for _ in range(2):  # repeated calls are bitwise identical
        out2 = torch.empty_like(q)
        lc2 = torch.full_like(lc, -1)
        z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out2, lc2, ws, gpu.status)
        gpu.check_status()
        assert torch.equal(lc2, lc) and torch.equal(out2.view(torch.int16), out.view(torch.int16))
    ref = Ref(wl, start + c.chunk)
    out = out.float().cpu().numpy()
    lc = lc.cpu().numpy()
    qf = q.float().cpu().numpy()
    rng = np.random.default_rng(1)
    tokens = sorted({0, 1, 127, 128, c.chunk - 1} | set(rng.choice(c.chunk, 6, replace=False).tolist()))
    for i in tokens:
        for h in range(c.n_q_heads):
            e_idx, e_counts, _, _ = ref.select(qf[i, h], 0, h, start + i, c.p)
            assert lc[i, h].tolist() == e_counts.tolist(), (i, h)
            o = ref.attend(qf[i, h], 0, h, e_idx)
            assert np.abs(out[i, h] - o).max() < TOL["bf16"], (i, h)


def test_top_scores_unsupported_geometry():
    """fp32 trees (and other geometries off the tensor-core path) are refused."""
    wl = W.make("tiny-f32-1k")
    gpu = Gpu(wl)
    c = wl.cfg
    q = torch.zeros(4, c.n_q_heads, c.head_dim, dtype=torch.float32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, 4, device=gpu.dev)
    with pytest.raises(z.ZhaError):
        z.zha_prefill_top_scores(gpu.cfg, gpu.cache, q, 0, 0, 0.95, None, None, ws, gpu.status)


@pytest.mark.slow
def test_prefill_full_size_sampled():
    """The full chunked-prefill workload (a 4096-token chunk after 1,048,576
    tokens, b = 4, L = 6, 257 top nodes for the last token), called as the
    benchmark calls it: zha_prefill_chunk over the whole chunk. 64 tokens x 16
    heads (1024 queries: the first and last token, both sides of the first
    tile edge 147/148, the rest seeded) against the oracle run over all host
    cores: level counts and outputs. Exact index lists through zha_select for
    the sampled tokens of two 148-token tiles (one CTA per unit, the prefill
    configuration) and of one-token calls (a cluster of CTAs per unit); then
    the tensor-core scores and certificates of the whole chunk."""
    from _oracle_pool import run_units

    wl = W.make("prefill-deep-1m-chunk4k")
    c = wl.cfg
    gpu = Gpu(wl)  # tree over the cached context
    start = c.n_tokens
    gpu.cache.seq_len.fill_(start + c.chunk)
    q = wl.queries(0).to(gpu.dev)
    out = torch.empty_like(q)
    lc = torch.full((c.chunk, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, c.chunk, device=gpu.dev)
    z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out, lc, ws, gpu.status)
    gpu.check_status()
    del ws
    torch.cuda.empty_cache()
    ref = Ref(wl, start + c.chunk)
    for kvh in range(c.n_kv_heads):
        compare_tree(gpu, ref, 0, kvh)  # the chunk's nodes, extended in place
    outn = out.float().cpu().numpy()
    lcn = lc.cpu().numpy()
    qf = q.float().cpu().numpy()
    rng = np.random.default_rng(4)
    edges = [0, 1, 147, 148, 2047, 3948, 4094, c.chunk - 1]
    rest = [int(i) for i in rng.permutation(c.chunk) if int(i) not in edges]
    tokens = sorted(edges + rest[:64 - len(edges)])
    # exact lists of the sampled tokens inside two 148-token tiles, and of two
    # one-token calls
    lists = {}
    for lo, nq in ((0, 148), (3948, 148), (0, 1), (c.chunk - 1, 1)):
        idx, n_idx, _, _ = gpu.select(q[lo:lo + nq].contiguous(), [0] * nq,
                                      [start + lo + i for i in range(nq)], c.p,
                                      start + c.chunk + 2)
        n_idx = n_idx.cpu().numpy()
        for i in tokens:
            if lo <= i < lo + nq:
                for h in range(c.n_q_heads):
                    lists[(nq, i, h)] = idx[i - lo, h, :n_idx[i - lo, h]].cpu().numpy()
        del idx
        torch.cuda.empty_cache()
    # oracle tasks: per KV head, the tokens split into 4 tasks (each rebuilds
    # the 1M-token tree)
    R = wl.R.float().cpu().numpy()
    tasks = []
    for kvh in range(c.n_kv_heads):
        for part in range(4):
            qs = [((i, h), qf[i, h], start + i, c.p, "full") for i in tokens[part::4]
                  for h in range(kvh * c.group, (kvh + 1) * c.group)]
            tasks.append({"unit": (0, kvh), "k": wl.K[0, kvh], "v": wl.V[0, kvh],
                          "dtype": c.dtype, "R": R, "n_tree": start + c.chunk, "b": c.block,
                          "L": c.levels, "cap": c.capacity, "queries": qs})
    n_list = 0
    for _, results, _ in run_units(tasks):
        for r in results:
            i, h = r["key"]
            assert lcn[i, h].tolist() == r["counts"].tolist(), (i, h)
            assert np.abs(outn[i, h] - r["out"]).max() < TOL["bf16"], (i, h)
            for nq in (148, 1):
                if (nq, i, h) in lists:
                    assert np.array_equal(lists[(nq, i, h)], r["idx"]), (nq, i, h)
                    n_list += 1
    assert n_list >= 16 * 8
    _check_top_scores(wl, gpu, ref, start, [0, 4095], 0.5)


PREFILL_GEOMETRIES = [
    # (context, chunk, block, levels, q heads, KV heads, head_dim, dtype)
    (20000, 200, 8, 4, 8, 2, 128, "bf16"),     # G = 4, 8 keep bytes per 64-key block
    (5000, 100, 2, 8, 16, 8, 128, "bf16"),     # G = 2, 32 keep bytes per block
    (12000, 64, 16, 3, 16, 2, 128, "bf16"),    # b = 16: 4 keep bytes per block
    (64, 200, 4, 3, 16, 2, 128, "bf16"),       # early tokens: 1 complete top node, then more
    (9000, 80, 4, 4, 16, 2, 64, "bf16"),       # d = 64: gather attention, canonical top level
    (3000, 60, 4, 3, 4, 1, 64, "f32"),         # fp32: gather attention, canonical top level
    (2, 100, 4, 3, 16, 2, 128, "bf16"),        # no complete top node for the first tokens
    (5000, 1, 4, 3, 16, 2, 128, "bf16"),       # one token: clusters of CTAs, 16 kept segments
]


@pytest.mark.parametrize("geom", PREFILL_GEOMETRIES, ids=lambda g: "-".join(map(str, g)))
def test_prefill_geometries(geom):
    """zha_prefill_chunk on geometries off the benchmark's: other block sizes
    and group sizes take other template instances of the tile attention and
    certificate kernels; d = 64 and fp32 take the gather attention and the
    canonical top level. Every (token, head) is checked against the oracle."""
    n, chunk, b, L, hq, hkv, d, dt = geom
    base = W.CONFIGS["prefill-deep-1m-chunk4k"]
    wl = W.Workload(base.scaled(n, chunk=chunk, block=b, levels=L, n_q_heads=hq, n_kv_heads=hkv,
                                head_dim=d, dtype=dt))
    c = wl.cfg
    gpu = Gpu(wl)
    start = c.n_tokens
    gpu.cache.seq_len.fill_(start + c.chunk)
    q = wl.queries(0).to(gpu.dev)
    out = torch.empty_like(q)
    lc = torch.full((c.chunk, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, c.chunk, device=gpu.dev)
    z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out, lc, ws, gpu.status)
    gpu.check_status()
    ref = Ref(wl, start + c.chunk)
    for kvh in range(c.n_kv_heads):
        compare_tree(gpu, ref, 0, kvh)
    out = out.float().cpu().numpy()
    lc = lc.cpu().numpy()
    qf = q.float().cpu().numpy()
    for i in range(c.chunk):
        for h in range(c.n_q_heads):
            e_idx, e_counts, _, _ = ref.select(qf[i, h], 0, h, start + i, c.p)
            assert lc[i, h].tolist() == e_counts.tolist(), (i, h)
            o = ref.attend(qf[i, h], 0, h, e_idx)
            assert np.abs(out[i, h] - o).max() < TOL[c.dtype], (i, h, np.abs(out[i, h] - o).max())


def test_tensor_core_wait_timeout_falls_back(monkeypatch):
    """The tensor-core completion wait is bounded (1 s). A test hook makes it
    wait for a barrier phase that never completes (the MMAs themselves finish;
    nothing faults or hangs): the call reports ZHA_ERR_TIMEOUT, certifies
    nothing, and zha_prefill_chunk still matches the oracle through the
    canonical top level. Without the hook the next call is clean again."""
    base = W.CONFIGS["prefill-deep-1m-chunk4k"]
    wl = W.Workload(base.scaled(16256, chunk=64))
    c = wl.cfg
    gpu = Gpu(wl)
    start = c.n_tokens
    gpu.cache.seq_len.fill_(start + c.chunk)
    z.zha_build_tree(gpu.cfg, gpu.cache)  # the tree covers the chunk too
    q = wl.queries(0).to(gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, c.chunk, device=gpu.dev)
    cert = torch.full((c.chunk, c.n_q_heads), -1, dtype=torch.int32, device=gpu.dev)

    monkeypatch.setenv("ZHA_TEST_TC_WAIT_PARITY", "1")
    gpu.status.zero_()
    z.zha_prefill_top_scores(gpu.cfg, gpu.cache, q, 0, start, c.p, None, cert, ws, gpu.status)
    torch.cuda.synchronize()
    assert int(gpu.status.item()) == z.ZHA_ERR_TIMEOUT
    assert (cert == 0).all()
    out = torch.empty_like(q)
    lc = torch.full((c.chunk, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    gpu.status.zero_()
    z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out, lc, ws, gpu.status)
    torch.cuda.synchronize()
    assert int(gpu.status.item()) == z.ZHA_ERR_TIMEOUT
    monkeypatch.delenv("ZHA_TEST_TC_WAIT_PARITY")

    ref = Ref(wl, start + c.chunk)
    outn = out.float().cpu().numpy()
    lcn = lc.cpu().numpy()
    qf = q.float().cpu().numpy()
    for i in (0, c.chunk // 2, c.chunk - 1):
        for h in range(c.n_q_heads):
            e_idx, e_counts, _, _ = ref.select(qf[i, h], 0, h, start + i, c.p)
            assert lcn[i, h].tolist() == e_counts.tolist(), (i, h)
            o = ref.attend(qf[i, h], 0, h, e_idx)
            assert np.abs(outn[i, h] - o).max() < TOL["bf16"], (i, h)

    gpu.status.zero_()
    z.zha_prefill_top_scores(gpu.cfg, gpu.cache, q, 0, start, c.p, None, cert, ws, gpu.status)
    gpu.check_status()
    assert float((cert == 1).float().mean()) > 0.3
