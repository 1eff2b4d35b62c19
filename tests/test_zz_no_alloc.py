"""zha_decode_noalloc (static device scratch, no workspace argument) against
zha_decode (caller workspace) through the C-ABI. Collected last on purpose:
it must also pass after every other test has run in the same process.

The static scratch keeps whatever the previous call left in it. So the
checked calls are interleaved with calls on other inputs (another step's
queries, another p): a stale candidate, counter or kept-list word read back
would make a checked call differ from zha_decode or from the oracle."""
import ctypes

import numpy as np
import pytest
import torch

from tree_indexed_sparse_zha_b200 import workloads as W

pytestmark = pytest.mark.gpu

STATIC_SCRATCH = 64 << 20


def _noalloc(z, gpu, q, p):
    c = gpu.c
    out = torch.empty_like(q)
    lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
    gpu.status.zero_()
    z.zha_decode_noalloc(gpu.cfg, gpu.cache, q, p, out, lc, gpu.status)
    gpu.check_status()
    return out.float().cpu().numpy(), lc.cpu().numpy()


def test_noalloc_decode_matches_decode_twice():
    from _harness import TOL, Gpu, Ref
    import tree_indexed_sparse_zha_b200 as z

    wl = W.make("decode-deep-32k")
    gpu = Gpu(wl)
    c = wl.cfg
    ref = Ref(wl, c.n_tokens)
    q0 = wl.queries(0).to(gpu.dev)
    q1 = wl.queries(1).to(gpu.dev)
    ref0 = gpu.decode(q0, c.p)
    ref1 = gpu.decode(q1, 0.8)
    qf = q0.float().cpu().numpy()
    counts0 = np.stack([ref.select(qf[0, h], 0, h, c.n_tokens - 1, c.p)[1]
                        for h in range(c.n_q_heads)])
    assert (ref0[1][0] == counts0).all()
    for _ in range(2):  # two checked calls in a row, each after a call on other inputs
        for q, p, (r_out, r_lc) in ((q1, 0.8, ref1), (q0, c.p, ref0)):
            out, lc = _noalloc(z, gpu, q, p)
            assert (lc == r_lc).all(), p
            err = np.abs(out - r_out).max()
            assert err <= TOL["bf16"], (p, err)
        assert (lc[0] == counts0).all()


def test_noalloc_near_the_scratch_limit():
    """The longest context of the 32K workload's geometry whose decode
    workspace still fits the static scratch: zha_decode_noalloc equals
    zha_decode there, on two calls with a shorter call between them."""
    from _harness import TOL, Gpu
    import tree_indexed_sparse_zha_b200 as z

    base = W.CONFIGS["decode-deep-32k"]

    def need(n):
        cfg = z.make_config(base.head_dim, base.block, base.levels, base.n_q_heads,
                            base.n_kv_heads, base.batch, n, base.torch_dtype)
        return z.zha_workspace_bytes(cfg, z.ZHA_OP_DECODE)

    lo, hi = 4096, 1 << 22  # need() grows with the capacity
    assert need(lo) <= STATIC_SCRATCH < need(hi)
    while hi - lo > 1024:
        mid = (lo + hi) // 2
        if need(mid) <= STATIC_SCRATCH:
            lo = mid
        else:
            hi = mid
    n = lo
    assert need(n) > 0.95 * STATIC_SCRATCH
    wl = W.make("decode-deep-32k", n_tokens=n)
    gpu = Gpu(wl)
    q = wl.queries(0).to(gpu.dev)
    r_out, r_lc = gpu.decode(q, wl.cfg.p)
    small = W.make("decode-deep-32k", n_tokens=20000)
    gs = Gpu(small)
    for _ in range(2):
        _noalloc(z, gs, small.queries(3).to(gs.dev), 0.5)
        out, lc = _noalloc(z, gpu, q, wl.cfg.p)
        assert (lc == r_lc).all()
        assert np.abs(out - r_out).max() <= TOL["bf16"]
    # one capacity step more is refused before any launch
    big = W.CONFIGS["decode-deep-32k"].scaled(hi)
    cfg = z.make_config(big.head_dim, big.block, big.levels, big.n_q_heads, big.n_kv_heads,
                        big.batch, big.capacity, big.torch_dtype)
    assert need(hi) > STATIC_SCRATCH
    st = z.lib().zha_decode_noalloc(ctypes.byref(cfg), ctypes.byref(gpu.cache.c()),
                                    ctypes.c_void_p(q.data_ptr()), 0.95,
                                    ctypes.c_void_p(q.data_ptr()), None, None, None)
    assert st == z.ZHA_ERR_WORKSPACE


def test_noalloc_rejects_geometry_beyond_static_scratch():
    from _harness import Gpu
    import tree_indexed_sparse_zha_b200 as z

    wl = W.make("decode-deep-32k", n_tokens=4096)
    gpu = Gpu(wl)
    c = W.CONFIGS["decode-deep-256k-b8"]
    big = z.make_config(c.head_dim, c.block, c.levels, c.n_q_heads, c.n_kv_heads, c.batch,
                        c.capacity, c.torch_dtype)
    need = ctypes.c_size_t(0)
    assert z.lib().zha_workspace_bytes(ctypes.byref(big), z.ZHA_OP_DECODE, 0,
                                       ctypes.byref(need)) == 0
    assert need.value > STATIC_SCRATCH
    q = torch.zeros(c.batch, c.n_q_heads, c.head_dim, dtype=torch.bfloat16, device=gpu.dev)
    out = torch.empty_like(q)
    st = z.lib().zha_decode_noalloc(ctypes.byref(big), ctypes.byref(gpu.cache.c()),
                                    ctypes.c_void_p(q.data_ptr()), 0.95,
                                    ctypes.c_void_p(out.data_ptr()), None, None, None)
    assert st == z.ZHA_ERR_WORKSPACE
