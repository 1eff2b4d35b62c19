"""The FP4 router variant on the GPU against the oracle.

zha_fp4_quantize_tree must give exactly oracle.fp4_round_rows of the tree's
rows (values and block exponents), also when it extends an existing copy
over newly completed nodes; zha_decode_fp4 must select exactly what the
oracle's traversal selects on the rounded tree (per-level counts and the
attended token lists, element by element), with outputs within 2e-2 of the
oracle's fp64 attention over that selection. Its drift from the canonical
selection is a property of the variant, checked loosely."""
import numpy as np
import pytest
import torch

import oracle
import tree_indexed_sparse_zha_b200 as z
from tree_indexed_sparse_zha_b200 import workloads as W

from _harness import TOL, Gpu, Ref

pytestmark = pytest.mark.gpu

MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _fp4_rows(gpu: Gpu, fp4: np.ndarray, seq: int, kvh: int, level: int):
    """Values and exponents of one unit's level from the 4-bit copy, decoded
    here from the documented format."""
    c = gpu.c
    nbytes, offs = z.zha_tree_layout(gpu.cfg)
    elems = nbytes // (2 if c.dtype == "bf16" else 4)
    codes_bytes = (elems // 2 + 255) // 256 * 256
    rows = c.capacity // c.block ** level
    e0 = offs[level - 1] + (seq * c.n_kv_heads + kvh) * rows * c.head_dim
    n = rows * c.head_dim
    b = fp4[e0 // 2:(e0 + n) // 2]
    nib = np.stack([b & 15, b >> 4], axis=1).reshape(-1)
    exps = fp4[codes_bytes:].view(np.int16)[e0 // 32:(e0 + n) // 32].astype(np.int64)
    val = MAG[nib & 7] * np.exp2(np.repeat(exps, 32).astype(np.float64))
    val = np.where(nib & 8, -val, val).astype(np.float32)
    return val.reshape(rows, c.head_dim), exps.reshape(rows, c.head_dim // 32)


def _compare_copy(gpu: Gpu, ref: Ref, fp4_t: torch.Tensor, units):
    fp4 = fp4_t.cpu().numpy()
    for s, kvh in units:
        tree = ref.tree(s, kvh)
        for l in range(1, gpu.c.levels + 1):
            rows = tree.level(l)
            got, ge = _fp4_rows(gpu, fp4, s, kvh, l)
            want, we = oracle.fp4_round_rows(rows)
            n = rows.shape[0]
            complete = ref.n // gpu.c.block ** l  # rows of nodes complete at the length
            assert np.array_equal(got[:complete], want[:complete]), (s, kvh, l)
            assert np.array_equal(ge[:complete], we[:complete]), (s, kvh, l)
            assert n >= complete


def test_quantize_matches_oracle_and_extends():
    wl = W.make("decode-deep-256k-b8", n_tokens=20000, batch=2)
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    fp4 = z.alloc_fp4_tree(gpu.cfg, gpu.dev)
    z.zha_fp4_quantize_tree(gpu.cfg, gpu.cache, fp4)
    torch.cuda.synchronize()
    units = [(s, k) for s in range(c.batch) for k in range(c.n_kv_heads)]
    _compare_copy(gpu, ref, fp4, units)
    # extend the tree and the copy over 200 appended tokens (completing nodes
    # up to level 3), against a copy quantized from scratch
    old = gpu.cache.seq_len.clone()
    gpu.cache.seq_len.add_(200)
    z.zha_extend_tree(gpu.cfg, gpu.cache, old, 200)
    z.zha_fp4_quantize_tree(gpu.cfg, gpu.cache, fp4, old)
    full = z.alloc_fp4_tree(gpu.cfg, gpu.dev)
    z.zha_fp4_quantize_tree(gpu.cfg, gpu.cache, full)
    torch.cuda.synchronize()
    n_new = c.n_tokens + 200
    nbytes, offs = z.zha_tree_layout(gpu.cfg)
    a, b = fp4.cpu().numpy(), full.cpu().numpy()
    elems = nbytes // 2
    codes_bytes = (elems // 2 + 255) // 256 * 256
    for s, kvh in units:
        for l in range(1, c.levels + 1):
            rows = c.capacity // c.block ** l
            done = n_new // c.block ** l
            e0 = offs[l - 1] + (s * c.n_kv_heads + kvh) * rows * c.head_dim
            e1 = e0 + done * c.head_dim
            assert np.array_equal(a[e0 // 2:e1 // 2], b[e0 // 2:e1 // 2]), (s, kvh, l)
            ea = a[codes_bytes:].view(np.int16)[e0 // 32:e1 // 32]
            eb = b[codes_bytes:].view(np.int16)[e0 // 32:e1 // 32]
            assert np.array_equal(ea, eb), (s, kvh, l)


def _fp4_parity(wl, p, seqs=None):
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    fp4 = z.alloc_fp4_tree(gpu.cfg, gpu.dev)
    z.zha_fp4_quantize_tree(gpu.cfg, gpu.cache, fp4)
    q = wl.queries(0).to(gpu.dev)
    out = torch.empty_like(q)
    lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    ws = gpu.decode_ws()
    z.zha_decode_fp4(gpu.cfg, gpu.cache, fp4, q, p, out, lc, ws, gpu.status)
    gpu.check_status()
    idx, n_idx = gpu.kept_lists(ws)
    idx, n_idx = idx.cpu().numpy(), n_idx.cpu().numpy()
    lc, out = lc.cpu().numpy(), out.float().cpu().numpy()
    t = c.n_tokens - 1
    qf = q.float().cpu().numpy()
    recall = []
    for s in (range(c.batch) if seqs is None else seqs):
        for kvh in range(c.n_kv_heads):
            t4 = oracle.fp4_tree(ref.tree(s, kvh))
            for h in range(kvh * c.group, (kvh + 1) * c.group):
                e_idx, e_counts, _, _ = oracle.select(qf[s, h], t4, t, p)
                assert lc[s, h].tolist() == e_counts.tolist(), (s, h, lc[s, h], e_counts)
                assert np.array_equal(idx[s, h, :n_idx[s, h]], e_idx), (s, h)
                o = ref.attend(qf[s, h], s, h, e_idx)
                assert np.abs(out[s, h] - o).max() < TOL[c.dtype], (s, h)
                canon, _, _, _ = ref.select(qf[s, h], s, h, t, p)
                recall.append(len(np.intersect1d(canon, e_idx)) / len(canon))
    return np.array(recall)


def test_decode_fp4_one_stream():
    """B = 1: two units, one stream."""
    r = _fp4_parity(W.make("decode-deep-32k"), 0.95)
    assert r.mean() > 0.9


def test_decode_fp4_grouped_ragged():
    """B = 8 (four unit groups on the library's streams), ragged lengths."""
    wl = W.make("decode-deep-256k-b8", n_tokens=24000)
    wl.seq_len[:] = torch.tensor([24000, 3000, 17777, 4096, 9001, 23999, 12345, 5000],
                                 dtype=torch.int32)
    c = wl.cfg
    gpu = Gpu(wl)
    ref = Ref(wl, c.n_tokens)
    fp4 = z.alloc_fp4_tree(gpu.cfg, gpu.dev)
    z.zha_fp4_quantize_tree(gpu.cfg, gpu.cache, fp4)
    q = wl.queries(2).to(gpu.dev)
    out = torch.empty_like(q)
    lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    ws = gpu.decode_ws()
    z.zha_decode_fp4(gpu.cfg, gpu.cache, fp4, q, 0.9, out, lc, ws, gpu.status)
    gpu.check_status()
    idx, n_idx = gpu.kept_lists(ws)
    idx, n_idx, lc = idx.cpu().numpy(), n_idx.cpu().numpy(), lc.cpu().numpy()
    out = out.float().cpu().numpy()
    qf = q.float().cpu().numpy()
    for s in (0, 1, 2, 7):
        t = int(wl.seq_len[s]) - 1
        for kvh in range(c.n_kv_heads):
            tree = oracle.build_tree(ref.K[s, kvh], t + 1, ref.R, c.block, c.levels, True,
                                     c.capacity)
            t4 = oracle.fp4_tree(tree)
            for h in range(kvh * c.group, (kvh + 1) * c.group):
                e_idx, e_counts, _, _ = oracle.select(qf[s, h], t4, t, 0.9)
                assert lc[s, h].tolist() == e_counts.tolist(), (s, h)
                assert np.array_equal(idx[s, h, :n_idx[s, h]], e_idx), (s, h)
                o = oracle.attend(qf[s, h], ref.K[s, kvh], ref.V[s, kvh], e_idx)
                assert np.abs(out[s, h] - o).max() < TOL[c.dtype], (s, h)


def test_decode_fp4_wide_tree():
    """b = 256, one level: the whole frontier is the top level."""
    r = _fp4_parity(W.make("decode-wide-256k-b8", n_tokens=16384, steps=1), 0.95, seqs=(0, 3))
    assert r.mean() > 0.95
