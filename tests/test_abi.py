"""The C-ABI library loads without a GPU, exports every declared entry point,
and rejects bad arguments on the host before any launch. CPU only."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "zha.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^(?:zha_status|const char\*)\s+(zha_\w+)\(", text, re.M)))


@pytest.fixture(scope="module")
def z():
    import __graft_entry__

    __graft_entry__.build()
    import tree_indexed_sparse_zha_b200 as z

    return z


def test_exports_every_declared_symbol(z):
    names = _declared_functions()
    assert len(names) == 19, names
    lib = z.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(z.EXPORTS)


def test_tree_layout_host_only(z):
    cfg = z.make_config(128, 4, 6, 16, 2, 8, 262400, torch.bfloat16)
    nbytes, offs = z.zha_tree_layout(cfg)
    rows = [262400 // 4 ** l for l in range(1, 7)]
    exp_offs = [sum(8 * 2 * r * 128 for r in rows[:i]) for i in range(6)]
    assert offs == exp_offs
    assert nbytes == 2 * sum(8 * 2 * r * 128 for r in rows)


def test_status_strings(z):
    assert z.status_string(0) == "ok"
    assert "capacity" in z.status_string(z.ZHA_ERR_CAPACITY)
    codes = [z.ZHA_ERR_INVALID_ARG, z.ZHA_ERR_UNSUPPORTED, z.ZHA_ERR_CUDA, z.ZHA_ERR_CAPACITY,
             z.ZHA_ERR_WORKSPACE, z.ZHA_ERR_TIMEOUT, z.ZHA_ERR_INTERNAL]
    texts = [z.status_string(c) for c in codes]
    assert len(set(texts)) == len(codes) and "unknown status" not in texts
    # device statuses are OR-ed flags: any set flag is named, the lowest first
    assert z.status_string(z.ZHA_ERR_TIMEOUT | z.ZHA_ERR_CAPACITY) == texts[3]
    assert z.status_string(1 << 20) == "unknown status"


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, 2), ("block", 3, 2), ("block", 48, 2), ("levels", 0, 1), ("levels", 9, 1),
    ("n_q_heads", 15, 1), ("n_q_heads", 12, 2), ("n_q_heads", 32, 2), ("batch", 0, 1), ("capacity", 0, 1),
    ("dtype", 7, 1), ("reserved", 1, 1),
])
def test_bad_geometry_rejected(z, field, value, code):
    cfg = z.make_config(128, 4, 6, 16, 2, 8, 262400, torch.bfloat16)
    setattr(cfg, field, value)
    n = ctypes.c_size_t(0)
    assert z.lib().zha_tree_layout(ctypes.byref(cfg), ctypes.byref(n), None) == code


def test_bad_arguments_rejected_before_launch(z):
    cfg = z.make_config(128, 4, 6, 16, 2, 1, 4096, torch.bfloat16)
    L = z.lib()
    # null cache / null pointers and p out of range never reach the device
    assert L.zha_build_tree(ctypes.byref(cfg), None, None) == z.ZHA_ERR_INVALID_ARG
    c = z.zha_cache(0, 0, 0, 0, 0)
    assert L.zha_build_tree(ctypes.byref(cfg), ctypes.byref(c), None) == z.ZHA_ERR_INVALID_ARG
    c = z.zha_cache(16, 16, 16, 16, 16)  # non-null dummies: p is checked first
    for p in (0.0, -0.5, float("nan")):
        assert L.zha_decode(ctypes.byref(cfg), ctypes.byref(c), ctypes.c_void_p(16), p,
                            ctypes.c_void_p(16), None, ctypes.c_void_p(16), 1 << 40, None,
                            None) == z.ZHA_ERR_INVALID_ARG
    # kept lists: null outputs, zero capacity and a short workspace
    ws_need = z.zha_workspace_bytes(cfg, z.ZHA_OP_DECODE)
    kl = L.zha_decode_kept_lists
    assert kl(ctypes.byref(cfg), ctypes.byref(c), ctypes.c_void_p(16), ws_need, None, 8,
              ctypes.c_void_p(16), None, None) == z.ZHA_ERR_INVALID_ARG
    assert kl(ctypes.byref(cfg), ctypes.byref(c), ctypes.c_void_p(16), ws_need,
              ctypes.c_void_p(16), 0, ctypes.c_void_p(16), None, None) == z.ZHA_ERR_INVALID_ARG
    assert kl(ctypes.byref(cfg), ctypes.byref(c), ctypes.c_void_p(16), ws_need - 1,
              ctypes.c_void_p(16), 8, ctypes.c_void_p(16), None, None) == z.ZHA_ERR_WORKSPACE
    # workspace too small
    assert L.zha_dense_decode(ctypes.byref(cfg), ctypes.byref(c), ctypes.c_void_p(16),
                              ctypes.c_void_p(16), ctypes.c_void_p(16), 1, None) == \
        z.ZHA_ERR_WORKSPACE


def test_fp4_router_host_side(z):
    cfg = z.make_config(128, 4, 6, 16, 2, 8, 262400, torch.bfloat16)
    nbytes, _ = z.zha_tree_layout(cfg)
    elems = nbytes // 2
    # 4-bit codes (rounded up to 256 bytes), then one int16 exponent per 32 elements
    assert z.zha_fp4_tree_bytes(cfg) == (elems // 2 + 255) // 256 * 256 + 2 * (elems // 32)
    L = z.lib()
    c = z.zha_cache(16, 16, 16, 16, 16)  # non-null dummies: never dereferenced here
    ws_need = z.zha_workspace_bytes(cfg, z.ZHA_OP_DECODE)
    args = (ctypes.c_void_p(16), 0.95, ctypes.c_void_p(16), None, ctypes.c_void_p(16), ws_need,
            None, None)
    # no FP4 copy, and head_dim 64 (the 4-bit scoring is written for 128)
    assert L.zha_decode_fp4(ctypes.byref(cfg), ctypes.byref(c), None, *args) == \
        z.ZHA_ERR_INVALID_ARG
    cfg64 = z.make_config(64, 4, 6, 16, 2, 8, 262400, torch.bfloat16)
    assert L.zha_decode_fp4(ctypes.byref(cfg64), ctypes.byref(c), ctypes.c_void_p(16), *args) == \
        z.ZHA_ERR_UNSUPPORTED
    assert L.zha_fp4_quantize_tree(ctypes.byref(cfg), ctypes.byref(c), None, None, None) == \
        z.ZHA_ERR_INVALID_ARG


def test_prefill_top_scores_rejected_before_launch(z):
    L = z.lib()
    c = z.zha_cache(16, 16, 16, 16, 16)  # non-null dummies: never dereferenced here

    def call(cfg, q, start, T, ws_bytes=1):
        return L.zha_prefill_top_scores(ctypes.byref(cfg), ctypes.byref(c), ctypes.c_void_p(q),
                                        0, start, T, 0.95, None, None, ctypes.c_void_p(256),
                                        ws_bytes, None, None)

    bf = z.make_config(128, 4, 3, 16, 2, 1, 40000, torch.bfloat16)
    assert call(bf, 256, 30000, 100) == z.ZHA_ERR_WORKSPACE        # valid, workspace too small
    assert call(bf, 258, 30000, 100) == z.ZHA_ERR_INVALID_ARG      # q not 16-byte aligned
    assert call(bf, 256, 39990, 100) == z.ZHA_ERR_INVALID_ARG      # chunk past the capacity
    assert call(bf, 256, 30000, 0) == z.ZHA_ERR_INVALID_ARG        # empty chunk
    f32 = z.make_config(128, 4, 3, 16, 2, 1, 40000, torch.float32)
    assert call(f32, 256, 30000, 100) == z.ZHA_ERR_UNSUPPORTED      # fp32: no tensor-core path
    one = z.make_config(128, 256, 1, 16, 2, 1, 40000, torch.bfloat16)
    assert call(one, 256, 30000, 100) == z.ZHA_ERR_UNSUPPORTED      # L = 1: no level below


def test_prefill_workspace_never_shrinks_with_the_chunk(z):
    # host-side sizing only (no device): a longer chunk never needs less
    cfg = z.make_config(128, 4, 6, 16, 2, 1, 1048576 + 4096, torch.bfloat16)
    sizes = [z.zha_workspace_bytes(cfg, z.ZHA_OP_PREFILL, T) for T in range(1, 401, 7)]
    assert all(b >= a for a, b in zip(sizes, sizes[1:])), sizes


def test_kernel_source_hash_is_stable():
    import importlib
    import sys

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()


def test_kernel_source_hash_ignores_comments_only():
    import importlib
    import sys

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    strip = bench.strip_c_comments
    base = 'int f(int a) { return a + 1; } // tail\nconst char* s = "//x /*y*/";\n'
    reworded = '/* lead */ int f(int a)  {\n  return a + 1; /* inline */ }\nconst char* s = "//x /*y*/";'
    assert strip(base) == strip(reworded)
    # literals that look like comments stay, and a code change shows
    assert '"//x /*y*/"' in strip(base)
    assert strip(base) != strip(base.replace("a + 1", "a + 2"))
    assert strip("char c = '\\'';  // q") == "char c = '\\'';"


def test_bench_selection_per_query():
    import importlib
    import sys

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    # b = 4, L = 2, n = 37: two complete top nodes (32 tokens) and a tail of 5
    lc = torch.tensor([[[2, 3], [1, 4]]], dtype=torch.int32)  # [B=1][Hq=2][L=2]
    r = bench.selection_per_query(lc, 4, 2, 37, 256)
    assert r["mean_kept_per_level"] == [1.5, 3.5]
    # (4 * 3 + 5) / 37 and (4 * 4 + 5) / 37
    assert abs(r["mean_selected_fraction"] - (17 / 37 + 21 / 37) / 2) < 1e-12
    # summary rows 2 + 4 * 2 and 2 + 4 * 1; K and V rows plus two 4-byte
    # index entries per selected token
    assert r["bytes_per_q_head_sum"] == (10 + 6) * 256 + (17 + 21) * (512 + 8)


def test_binding_refuses_host_tensors(z):
    # every pointer the library takes is device memory: a host tensor is
    # refused in the binding, before any call into the library
    with pytest.raises(ValueError, match="device"):
        z._ptr(torch.zeros(4))
    cfg = z.make_config(64, 4, 3, 1, 1, 1, 1024, torch.float32)
    host = z.Cache(torch.zeros(1, 1, 1024, 64), torch.zeros(1, 1, 1024, 64),
                   torch.zeros(16, 64), torch.zeros(8), torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="cache.k"):
        z.zha_build_tree(cfg, host)
    assert z._ptr(None) is None


def test_bench_clock_sampler_parses_nvidia_smi(tmp_path, monkeypatch):
    import importlib
    import sys
    import time

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n"
                    "echo '0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active'\n"
                    "echo '0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "echo '0, 1900, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "echo 'garbled line'\n"
                    "exec sleep 30\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}:{os.environ['PATH']}")
    s = bench.ClockSampler(0)
    s.start()
    deadline = time.time() + 10
    while len(s.lines) < 4 and time.time() < deadline:
        time.sleep(0.05)
    r = s.stop()
    assert r == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def _ptxas_frame(report: str, mangled_part: str):
    """(stack frame bytes, spill store bytes) of the kernel whose mangled name
    contains mangled_part, from a ptxas -v report."""
    lines = report.splitlines()
    for i, ln in enumerate(lines):
        if "Function properties for" in ln and mangled_part in ln and i + 1 < len(lines):
            m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores", lines[i + 1])
            if m:
                return int(m.group(1)), int(m.group(2))
    return None


def test_traversal_stack_frame_stays_small(z):
    # The traversal hands its parameter block by reference to non-inlined
    # helpers; unless the parameter is grid-constant, every thread copies the
    # whole block to its stack at launch (a 784-byte frame for the bf16,
    # d = 128, 8-head instance, against 304 bytes with it).
    from tree_indexed_sparse_zha_b200 import build as B

    path = B.ptxas_report_path(os.path.join(B.CSRC, "traverse.cu"))
    if not os.path.exists(path):
        B.build(force=True)
    with open(path) as f:
        report = f.read()
    frame = _ptxas_frame(report, "traverse_kernelI13__nv_bfloat16Li128ELi8E")
    assert frame is not None, "traverse_kernel<bf16, 128, 8> missing from the ptxas report"
    assert frame[0] <= 384 and frame[1] <= 64, frame


def test_bench_decode_step_bytes():
    import importlib
    import sys

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    # by hand: 2 units, b = 4, 10 kept level-1 nodes, a tail of 3 tokens,
    # 100 summary rows, 16 queries, 256-byte rows
    sel, att, kv = bench.decode_step_bytes(100, 10, 4, 3, 2, 16, 256)
    assert kv == 10 * 4 + 2 * (1 + 3)
    assert sel == 100 * 256 + 10 * 4 + 16 * 256  # queries read; outputs belong to attention
    assert att == kv * 512 + 10 * 4 + 2 * 16 * 256
    # the counts of a measured 256K decode step (16 units, 128 queries) give
    # the bytes that step reported
    sel, att, kv = bench.decode_step_bytes(1397720, 1048300, 4, 205, 16, 128, 256)
    assert kv == 4196496 and sel + att == 2514939744 - 128 * 256


def test_bench_prefill_selection():
    import importlib
    import sys

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    # by hand: b = 4, L = 2 (top nodes of 16 tokens), chunk tokens at positions
    # 30, 31, 32 (31, 32, 33 visible tokens: tails of 15, 0 and 1), 2 heads,
    # kept counts top level first
    lc = torch.tensor([[[1, 2], [1, 3]], [[2, 4], [2, 0]], [[1, 1], [2, 1]]], dtype=torch.int32)
    got = bench.prefill_selection(lc, 4, 2, 30)
    assert got["mean_kept_per_level"] == [1.5, round(11 / 6, 3)]
    sel_frac = [23 / 31, 27 / 31, 16 / 32, 0 / 32, 5 / 33, 5 / 33]
    assert abs(got["mean_selected_fraction"] - sum(sel_frac) / 6) < 1e-12
