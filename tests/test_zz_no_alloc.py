"""zha_decode_noalloc (static device scratch, no workspace argument) against
zha_decode (caller workspace) through the C-ABI. Collected last on purpose:
it must also pass after every other test has run in the same process."""
import ctypes

import pytest
import torch

from tree_indexed_sparse_zha_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_decode_twice():
    from _harness import TOL, Gpu
    import tree_indexed_sparse_zha_b200 as z

    wl = W.make("decode-deep-32k")
    gpu = Gpu(wl)
    c = wl.cfg
    q = wl.queries(0).to(gpu.dev)
    ref_out, ref_lc = gpu.decode(q, c.p)
    for _ in range(2):  # two calls in a row reuse the same static scratch
        out = torch.empty_like(q)
        lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=gpu.dev)
        gpu.status.zero_()
        z.zha_decode_noalloc(gpu.cfg, gpu.cache, q, c.p, out, lc, gpu.status)
        gpu.check_status()
        assert (lc.cpu().numpy() == ref_lc).all()
        err = (out.float().cpu().numpy() - ref_out).__abs__().max()
        assert err <= TOL["bf16"], err


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
    assert need.value > (64 << 20)
    q = torch.zeros(c.batch, c.n_q_heads, c.head_dim, dtype=torch.bfloat16, device=gpu.dev)
    out = torch.empty_like(q)
    st = z.lib().zha_decode_noalloc(ctypes.byref(big), ctypes.byref(gpu.cache.c()),
                                    ctypes.c_void_p(q.data_ptr()), 0.95,
                                    ctypes.c_void_p(out.data_ptr()), None, None, None)
    assert st == z.ZHA_ERR_WORKSPACE
