"""zha_decode runs a step's (sequence, KV head) units in up to 4 groups on
streams of the library's own. Every kernel computes per unit what the
one-stream order (zha_decode_select then zha_decode_attend, or
zha_decode_noalloc) computes, so outputs, level counts and attended token
lists must agree bit for bit -- for uneven groups, ragged lengths (one
sequence below its first complete top node) and inside a CUDA graph."""
import numpy as np
import pytest
import torch

import tree_indexed_sparse_zha_b200 as z
from tree_indexed_sparse_zha_b200 import workloads as W

from _harness import Gpu

pytestmark = pytest.mark.gpu


def _one_stream(gpu: Gpu, q, p, ws):
    c = gpu.c
    out = torch.empty_like(q)
    lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    z.zha_decode_select(gpu.cfg, gpu.cache, q, p, lc, ws, gpu.status)
    z.zha_decode_attend(gpu.cfg, gpu.cache, q, out, ws)
    gpu.check_status()
    idx, n_idx = gpu.kept_lists(ws)
    return out, lc, idx, n_idx


def _grouped(gpu: Gpu, q, p, ws):
    c = gpu.c
    out = torch.empty_like(q)
    lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    z.zha_decode(gpu.cfg, gpu.cache, q, p, out, lc, ws, gpu.status)
    gpu.check_status()
    idx, n_idx = gpu.kept_lists(ws)
    return out, lc, idx, n_idx


def _same(a, b):
    out_a, lc_a, idx_a, n_a = a
    out_b, lc_b, idx_b, n_b = b
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(lc_a, lc_b)
    assert torch.equal(n_a, n_b)
    for s in range(n_a.shape[0]):
        for h in range(n_a.shape[1]):
            n = int(n_a[s, h])
            assert torch.equal(idx_a[s, h, :n], idx_b[s, h, :n]), (s, h)


@pytest.mark.parametrize("batch", [2, 3, 5, 8])
def test_groups_equal_one_stream_ragged(batch):
    """Groups of 1..4 (uneven for 3 and 5 sequences): sequence lengths from
    3000 tokens (no complete top node: token 0 and the tail only) to 24000."""
    wl = W.make("decode-deep-256k-b8", n_tokens=24000, batch=batch)
    lens = [24000, 3000, 17777, 4096, 9001, 23999, 12345, 5000][:batch]
    wl.seq_len[:] = torch.tensor(lens, dtype=torch.int32)
    gpu = Gpu(wl)
    ws = gpu.decode_ws()
    for step, p in ((1, 0.95), (2, 0.5)):
        q = wl.queries(step).to(gpu.dev)
        a = _one_stream(gpu, q, p, ws)
        b = _grouped(gpu, q, p, ws)
        _same(a, b)
        assert int(b[1][1, 0, 0]) == 0  # the short sequence has no top node


def test_grouped_in_cuda_graph_matches_eager():
    """Extension + zha_decode captured once in a CUDA graph and replayed over
    four appended tokens (lengths and queries copied into the graph's input
    buffers) give what the eager one-stream calls give on a twin cache."""
    wl = W.make("decode-deep-256k-b8", n_tokens=20000)
    c = wl.cfg
    g_gpu, e_gpu = Gpu(wl), Gpu(wl)
    ws_g, ws_e = g_gpu.decode_ws(), e_gpu.decode_ws()
    old_st = g_gpu.cache.seq_len.clone()
    q_st = wl.queries(1).to(g_gpu.dev)
    out_g = torch.empty_like(q_st)
    lc_g = torch.zeros(c.batch, c.n_q_heads, c.levels, dtype=torch.int32, device=g_gpu.dev)

    def body():
        z.zha_extend_tree(g_gpu.cfg, g_gpu.cache, old_st, 1)
        z.zha_decode(g_gpu.cfg, g_gpu.cache, q_st, c.p, out_g, lc_g, ws_g, g_gpu.status)

    # an eager call first creates the library's streams (outside any capture)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        z.zha_decode(g_gpu.cfg, g_gpu.cache, q_st, c.p, out_g, lc_g, ws_g, g_gpu.status)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        body()
    torch.cuda.synchronize()
    for step in range(1, 5):
        q = wl.queries(step).to(g_gpu.dev)
        old_st.copy_(g_gpu.cache.seq_len)
        g_gpu.cache.seq_len.add_(1)
        q_st.copy_(q)
        graph.replay()
        g_gpu.check_status()
        old_e = e_gpu.cache.seq_len.clone()
        e_gpu.cache.seq_len.add_(1)
        z.zha_extend_tree(e_gpu.cfg, e_gpu.cache, old_e, 1)
        out_e, lc_e, _, _ = _one_stream(e_gpu, q, c.p, ws_e)
        assert torch.equal(out_g.view(torch.int16), out_e.view(torch.int16)), step
        assert torch.equal(lc_g, lc_e), step
    assert torch.equal(g_gpu.cache.tree, e_gpu.cache.tree)
