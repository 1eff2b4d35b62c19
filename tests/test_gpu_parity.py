"""CUDA path vs the CPU oracle, through the C-ABI.

Bar: summary trees, selected index sets and per-level kept counts bit-exact;
attention outputs within max-abs 2e-2 (bf16 I/O, fp32 accumulation) or 1e-5
(fp32 mode) of the oracle's fp64 attention over the oracle's own selection."""
import numpy as np
import pytest
import torch

from tree_indexed_sparse_zha_b200 import workloads as W

from _harness import TOL, Gpu, Ref, compare_tree

pytestmark = pytest.mark.gpu


def _decode_parity(wl, step_q, p, n_tokens, units=None, heads=None):
    """zha_decode + zha_select + zha_attend on the current cache state vs oracle."""
    c = wl.cfg
    gpu = _decode_parity.gpu
    ref = _decode_parity.ref
    q = step_q.to(gpu.dev)
    out, lc, kidx, kn = gpu.decode(q, p, lists=True)
    kidx = kidx.cpu().numpy()
    kn = kn.cpu().numpy()
    t = n_tokens - 1
    qf = q.float().cpu().numpy()
    seqs = range(c.batch) if units is None else units
    hs = range(c.n_q_heads) if heads is None else heads
    cap = n_tokens + 2
    idx, n_idx, lcs, qs = gpu.select(q, list(range(c.batch)), [t] * c.batch, p, cap)
    att = gpu.attend(q, qs, idx, n_idx)
    idx = idx.cpu().numpy()
    n_idx = n_idx.cpu().numpy()
    lcs = lcs.cpu().numpy()
    flagged = 0
    for s in seqs:
        for h in hs:
            e_idx, e_counts, _, tie = ref.select(qf[s, h], s, h, t, p)
            flagged += tie
            assert lc[s, h].tolist() == e_counts.tolist(), (s, h, lc[s, h], e_counts)
            # the set the decode step's attention read, element by element
            assert kn[s, h] == len(e_idx), (s, h, kn[s, h], len(e_idx))
            assert np.array_equal(kidx[s, h, :kn[s, h]], e_idx), (s, h)
            assert lcs[s, h].tolist() == e_counts.tolist()
            assert n_idx[s, h] == len(e_idx)
            assert np.array_equal(idx[s, h, :n_idx[s, h]], e_idx), (s, h)
            o = ref.attend(qf[s, h], s, h, e_idx)
            tol = TOL[c.dtype]
            assert np.abs(out[s, h] - o).max() < tol, (s, h, np.abs(out[s, h] - o).max())
            assert np.abs(att[s, h] - o).max() < tol
    return flagged


def _run_decode_case(wl, p=None, units=None, heads=None, check_tree_units=None):
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    _decode_parity.gpu, _decode_parity.ref = gpu, ref
    for (s, k) in (check_tree_units or [(s, k) for s in range(c.batch)
                                        for k in range(c.n_kv_heads)]):
        compare_tree(gpu, ref, s, k)
    return _decode_parity(wl, wl.queries(0), c.p if p is None else p, c.n_tokens, units, heads)


def test_tiny_f32():
    _run_decode_case(W.make("tiny-f32-1k"))


def test_decode_deep_32k():
    _run_decode_case(W.make("decode-deep-32k"))


@pytest.mark.parametrize("n", [300, 4095, 4096, 4097, 9000])
def test_ragged_lengths(n):
    # fewer tokens than one top node (dense), exactly one, one plus a tail
    _run_decode_case(W.make("decode-deep-32k", n_tokens=n))


def test_tiny_p_sweep():
    wl = W.make("tiny-f32-1k")
    for p in (1e-6, 0.3, 0.8, 0.999, 1.0):
        _run_decode_case(wl, p=p)


def test_decode_deep_256k_scaled_incremental():
    """Scaled copy of the 256K decode run: 8 sequences, extend + decode every step."""
    wl = W.make("decode-deep-256k-b8", n_tokens=16384 + 4090, steps=24)
    c = wl.cfg
    gpu = Gpu(wl)
    z = __import__("tree_indexed_sparse_zha_b200")
    final_n = c.n_tokens + c.steps
    ref = Ref(wl, final_n)
    _decode_parity.gpu, _decode_parity.ref = gpu, ref
    old = gpu.cache.seq_len.clone()
    for step in range(1, c.steps + 1):
        old.copy_(gpu.cache.seq_len)
        gpu.cache.seq_len.add_(1)
        z.zha_extend_tree(gpu.cfg, gpu.cache, old, 1)
        n = c.n_tokens + step
        if step in (1, 6, 7, 23, 24):  # 16384+4096 = 20480 completes a top node at step 6
            _decode_parity(wl, wl.queries(step), c.p, n)
    torch.cuda.synchronize()
    for s in range(c.batch):
        for k in range(c.n_kv_heads):
            compare_tree(gpu, ref, s, k)


def test_decode_wide_scaled_p_sweep():
    wl = W.make("decode-wide-256k-b8", n_tokens=16384 + 100)
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    _decode_parity.gpu, _decode_parity.ref = gpu, ref
    compare_tree(gpu, ref, 0, 0)
    compare_tree(gpu, ref, 7, 1)
    q = wl.queries(0)
    for p in c.p_sweep:
        _decode_parity(wl, q, p, c.n_tokens)
    # p = 1 keeps everything: the sparse path equals the dense kernel
    out1, _ = gpu.decode(q.to(gpu.dev), 1.0)
    dense = gpu.dense(q.to(gpu.dev))
    assert np.abs(out1 - dense).max() < TOL["bf16"]


def test_prefill_scaled():
    """Scaled chunked prefill: a 256-token chunk whose middle completes a top
    node (positions 16256..16511; top node 3 ends at 16383), causal."""
    base = W.CONFIGS["prefill-deep-1m-chunk4k"]
    wl = W.Workload(base.scaled(16256, chunk=256))
    c = wl.cfg
    gpu = Gpu(wl)  # tree over the first 16384 tokens
    z = __import__("tree_indexed_sparse_zha_b200")
    start = c.n_tokens
    gpu.cache.seq_len.fill_(start + c.chunk)
    q = wl.queries(0).to(gpu.dev)
    out = torch.empty_like(q)
    lc = torch.full((c.chunk, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_PREFILL, c.chunk, device=gpu.dev)
    z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out, lc, ws, gpu.status)
    gpu.check_status()
    # repeated calls on the same tree are bitwise identical (the cut is exact)
    for _ in range(4):
        out2 = torch.empty_like(q)
        lc2 = torch.full_like(lc, -1)
        gpu.cache.seq_len.fill_(start + c.chunk)
        z.zha_prefill_chunk(gpu.cfg, gpu.cache, q, 0, start, c.p, out2, lc2, ws, gpu.status)
        gpu.check_status()
        assert torch.equal(lc2, lc) and torch.equal(out2.view(torch.int16), out.view(torch.int16))
    ref = Ref(wl, start + c.chunk)
    compare_tree(gpu, ref, 0, 0)
    compare_tree(gpu, ref, 0, 1)
    out = out.float().cpu().numpy()
    lc = lc.cpu().numpy()
    qf = q.float().cpu().numpy()
    rng = np.random.default_rng(0)
    tokens = sorted(set([0, 1, 126, 127, 128, c.chunk - 2, c.chunk - 1])
                    | set(rng.choice(c.chunk, 12, replace=False).tolist()))
    for i in tokens:
        for h in range(c.n_q_heads):
            e_idx, e_counts, _, _ = ref.select(qf[i, h], 0, h, start + i, c.p)
            assert lc[i, h].tolist() == e_counts.tolist(), (i, h)
            o = ref.attend(qf[i, h], 0, h, e_idx)
            assert np.abs(out[i, h] - o).max() < TOL["bf16"], (i, h)


def test_capacity_overflow_sets_status():
    wl = W.make("decode-deep-32k", n_tokens=5000)
    gpu = Gpu(wl)
    q = wl.queries(0).to(gpu.dev)
    gpu.select(q, [0], [4999], 0.95, 5001)  # fits
    z = __import__("tree_indexed_sparse_zha_b200")
    idx = torch.zeros(1, 16, 8, dtype=torch.int32, device=gpu.dev)
    n_idx = torch.zeros(1, 16, dtype=torch.int32, device=gpu.dev)
    ws = z.alloc_workspace(gpu.cfg, z.ZHA_OP_SELECT, 1, device=gpu.dev)
    qs = torch.zeros(1, dtype=torch.int32, device=gpu.dev)
    qp = torch.full((1,), 4999, dtype=torch.int32, device=gpu.dev)
    z.zha_select(gpu.cfg, gpu.cache, q, qs, qp, 0.95, idx, n_idx, None, ws, gpu.status)
    torch.cuda.synchronize()
    assert int(gpu.status.item()) & z.ZHA_ERR_CAPACITY
    assert (n_idx > 8).all()


def test_dense_decode_vs_oracle():
    """zha_dense_decode (flash-decoding over every key [0, t]) against the
    oracle's fp64 softmax attention over the same keys, all 16 heads, on the
    32K workload and on a ragged length with no complete top node."""
    import oracle

    for n in (32768, 3001):
        wl = W.make("decode-deep-32k", n_tokens=n)
        c = wl.cfg
        gpu = Gpu(wl, build=False)
        q = wl.queries(0)
        out = gpu.dense(q.to(gpu.dev))
        qf = q.float().numpy()
        K, V = wl.K.float().numpy(), wl.V.float().numpy()
        for h in range(c.n_q_heads):
            kvh = h // c.group
            o = oracle.dense(qf[0, h], K[0, kvh], V[0, kvh], n - 1)
            assert np.abs(out[0, h] - o).max() < TOL["bf16"], (n, h)


def test_zero_query_all_ties():
    """q = 0: every node of a level has the same score, so each cut is decided
    purely by the lower-node-index rule (ordered tie ranks)."""
    wl = W.make("decode-deep-32k", n_tokens=20000)
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    _decode_parity.gpu, _decode_parity.ref = gpu, ref
    q = torch.zeros_like(wl.queries(0))
    for p in (0.3, 0.95):
        _decode_parity(wl, q, p, c.n_tokens)


def test_decode_clustered_keys_narrowed_groups():
    """Decode (B = 1, 131K context) over keys that form one tight cluster
    (a common vector plus 0.01 noise) with one far-off key every 256 tokens:
    the far keys stretch each level's score range, so the cluster's
    candidates crowd into a few first-pass buckets and, at level 1, the
    crossing bucket holds thousands of them with distinct keys. The cut then
    narrows it by key digits before ranking. Counts and attended sets must
    equal the oracle's for every head."""
    wl = W.make("decode-deep-32k", n_tokens=131072)
    c = wl.cfg
    g = torch.Generator().manual_seed(3)
    n = c.n_tokens
    for kvh in range(c.n_kv_heads):
        v = torch.randn(c.head_dim, generator=g)
        keys = v + 0.01 * torch.randn(n, c.head_dim, generator=g)
        keys[::256] = 3.0 * torch.randn(keys[::256].shape, generator=g)
        wl.K[0, kvh, :n] = keys.to(c.torch_dtype)
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    _decode_parity.gpu, _decode_parity.ref = gpu, ref
    for p in (0.5, 0.95):
        _decode_parity(wl, wl.queries(0), p, c.n_tokens)


def test_decode_long_context_large_frontier():
    """Decode at 400K context (B = 1) with p = 0.999: the level-1 frontier of a
    head exceeds what the cut keeps bucket bytes for in shared memory, and the
    kept list one level up exceeds its shared copy, so the cut streams its
    parents and scores from global memory. Checked head by head against the
    oracle."""
    wl = W.make("decode-deep-32k", n_tokens=400000)
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    _decode_parity.gpu, _decode_parity.ref = gpu, ref
    _decode_parity(wl, wl.queries(0), 0.999, c.n_tokens)


def test_select_one_cta_narrowed_groups():
    """148 queries (one CTA per (query, KV head) unit, as a prefill tile runs)
    at 131K context, small-norm queries and p = 0.5 / 0.95: the crossing
    first-pass buckets hold hundreds of candidates, so a head's group is
    narrowed by key-digit passes before its owner gathers it, and the other
    members of the bucket (above and below the group) keep or lose their place
    by key. Index lists must equal the oracle's exactly."""
    wl = W.make("decode-deep-32k", n_tokens=131072)
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    nq = 148
    g = torch.Generator().manual_seed(7)
    q = (0.05 * torch.randn(nq, c.n_q_heads, c.head_dim, generator=g)).to(c.torch_dtype)
    pos = [c.n_tokens - 1 - i for i in range(nq)]
    qf = q.float().numpy()
    for p in (0.5, 0.95):
        idx, n_idx, lcs, _ = gpu.select(q.to(gpu.dev), [0] * nq, pos, p, c.n_tokens + 2)
        n_idx = n_idx.cpu().numpy()
        lcs = lcs.cpu().numpy()
        for i in (0, 1, 73, 147):
            rows = idx[i].cpu().numpy()
            for h in range(c.n_q_heads):
                e_idx, e_counts, _, _ = ref.select(qf[i, h], 0, h, pos[i], p)
                assert lcs[i, h].tolist() == e_counts.tolist(), (p, i, h)
                assert n_idx[i, h] == len(e_idx), (p, i, h, n_idx[i, h], len(e_idx))
                assert np.array_equal(rows[h, :n_idx[i, h]], e_idx), (p, i, h)
        del idx


@pytest.mark.parametrize("dtype,d,b,L,n", [
    ("f32", 64, 64, 2, 64 * 64 * 3 + 70),     # two levels, ragged tail
    ("bf16", 128, 96, 1, 96 * 40 + 5),        # b not a power of two
    ("bf16", 64, 128, 2, 128 * 128 + 300),
    ("f32", 128, 256, 1, 256 * 30 + 17),      # the widest staged kernel, fp32 rows
    ("bf16", 128, 512, 1, 512 * 9 + 100),     # one CTA of b threads per node
])
def test_tree_wide_blocks_ragged_and_extend(dtype, d, b, L, n):
    """Summary trees with wide blocks against the oracle, bit for bit: built
    over ragged lengths (3 sequences, 2 KV heads), then extended by a few
    hundred tokens per sequence (nodes completed by the new tokens only)."""
    import oracle
    import tree_indexed_sparse_zha_b200 as z
    cfg = W.WorkloadConfig(f"tree-b{b}", 5, dtype, 3, 4, 2, d, n, b, L, 0.95, (1, 2), steps=600)
    wl = W.Workload(cfg)
    gpu = Gpu(wl, build=False)
    lens0 = [n - 3 * b - 1, n, b ** L - 1]
    gpu.cache.seq_len.copy_(torch.tensor(lens0, dtype=torch.int32))
    z.zha_build_tree(gpu.cfg, gpu.cache)
    K = wl.K.float().numpy()
    R = wl.R.numpy()

    def check(lens):
        torch.cuda.synchronize()
        for s in range(cfg.batch):
            for kvh in range(cfg.n_kv_heads):
                got = gpu.tree_unit(s, kvh)
                exp = oracle.build_tree(K[s, kvh], lens[s], R, b, L, dtype == "bf16", cfg.capacity)
                for l in range(1, L + 1):
                    m = lens[s] // b ** l
                    a, e = got[l - 1][:m], exp.level(l)[:m]
                    assert np.array_equal(a.view(np.uint32), e.view(np.uint32)), (s, kvh, l)

    check(lens0)
    old = gpu.cache.seq_len.clone()
    lens1 = [x + 600 for x in lens0]
    gpu.cache.seq_len.copy_(torch.tensor(lens1, dtype=torch.int32))
    z.zha_extend_tree(gpu.cfg, gpu.cache, old, 600)
    check(lens1)
