"""CPU oracle for the ZHA hot path (tree build, top-p traversal, sparse attention).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference leg may import this package. It shares
no code with the CUDA path and never imports it.

The arithmetic lives in ``zha_oracle.c`` (plain single-threaded C, built with
``-O2 -ffp-contract=off``); this module only marshals numpy arrays through
ctypes. See the C file's header for the passages each function follows
(lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
paragraphs 1-2) and for the canonical fp32 arithmetic.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zha_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libzha_oracle.so")

_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u64p = ctypes.POINTER(ctypes.c_uint64)
_intp = ctypes.POINTER(ctypes.c_int)


def _cpu_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    return " fma " in (line.strip() + " ")
    except OSError:
        pass
    return False


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libzha_oracle.so``.

    ``-mfma`` only lets gcc inline the ``fmaf`` calls; the rounding is the same
    with or without it (fmaf is exactly rounded either way).
    """
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    flags = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
    if _cpu_has_fma():
        flags.append("-mfma")
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *flags, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        L.zo_exp_c.argtypes = [ctypes.c_float]
        L.zo_exp_c.restype = ctypes.c_float
        L.zo_dot.argtypes = [_f32p, _f32p, ctypes.c_int]
        L.zo_dot.restype = ctypes.c_float
        L.zo_round_bf16.argtypes = [ctypes.c_float]
        L.zo_round_bf16.restype = ctypes.c_float
        L.zo_build_node.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, _f32p, ctypes.c_int, _f32p]
        L.zo_build_node.restype = None
        L.zo_build_node_f64.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, _f32p, _f64p]
        L.zo_build_node_f64.restype = None
        L.zo_build_tree.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int, _f32p, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, _f32p, _i64p]
        L.zo_build_tree.restype = ctypes.c_int64
        L.zo_p_fixed.argtypes = [ctypes.c_double]
        L.zo_p_fixed.restype = ctypes.c_uint64
        L.zo_cut.argtypes = [_f32p, _i64p, ctypes.c_int64, ctypes.c_uint64, _i64p, _u64p, _u64p,
                             _intp]
        L.zo_cut.restype = ctypes.c_int64
        L.zo_score.argtypes = [_f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.zo_score.restype = ctypes.c_float
        L.zo_select.argtypes = [_f32p, ctypes.c_int, _f32p, _i64p, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int64, ctypes.c_uint64, _i32p, ctypes.c_int64, _i32p,
                                _i64p, _intp]
        L.zo_select.restype = ctypes.c_int64
        L.zo_select_f64.argtypes = [_f32p, ctypes.c_int, _f32p, _i64p, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int64, ctypes.c_double, _i32p, ctypes.c_int64, _i32p,
                                    _f64p]
        L.zo_select_f64.restype = ctypes.c_int64
        L.zo_fp4_round_rows.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int, _f32p, _i32p]
        L.zo_fp4_round_rows.restype = None
        L.zo_attend_f64.argtypes = [_f32p, ctypes.c_int, _f32p, _f32p, _i32p, ctypes.c_int64,
                                    _f64p]
        L.zo_attend_f64.restype = None
        _lib = L
    return _lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)


# ---------------------------------------------------------------------------
# scalar canonical helpers (exposed for the pins)
# ---------------------------------------------------------------------------

def exp_c(x: float) -> float:
    return float(lib().zo_exp_c(ctypes.c_float(x)))


def round_bf16(x: float) -> float:
    return float(lib().zo_round_bf16(ctypes.c_float(x)))


def p_fixed(p: float) -> int:
    """p_q = floor(p * 2^32 + 0.5): the fixed-point form of the coverage p."""
    return int(lib().zo_p_fixed(ctypes.c_double(p)))


def dot(a, x) -> float:
    a = _f32(a)
    x = _f32(x)
    return float(lib().zo_dot(_ptr(a, _f32p), _ptr(x, _f32p), a.shape[0]))


def score(q, s, level: int, b: int) -> float:
    q = _f32(q)
    s = _f32(s)
    return float(lib().zo_score(_ptr(q, _f32p), _ptr(s, _f32p), q.shape[0], level, b))


# ---------------------------------------------------------------------------
# summaries
# ---------------------------------------------------------------------------

def build_node(children, R, store_bf16: bool = False) -> np.ndarray:
    ch = _f32(children)
    R = _f32(R)
    b, d = ch.shape
    out = np.empty(d, dtype=np.float32)
    lib().zo_build_node(_ptr(ch, _f32p), b, d, _ptr(R, _f32p), int(store_bf16), _ptr(out, _f32p))
    return out


def build_node_f64(children, R) -> np.ndarray:
    ch = _f32(children)
    R = _f32(R)
    b, d = ch.shape
    out = np.empty(d, dtype=np.float64)
    lib().zo_build_node_f64(_ptr(ch, _f32p), b, d, _ptr(R, _f32p), _ptr(out, _f64p))
    return out


def level_row_offsets(n_cap: int, b: int, L: int) -> Tuple[np.ndarray, int]:
    """Row offset of each level (1..L) in a packed per-unit tree, and the total
    row count. Level l holds floor(n_cap / b^l) rows."""
    offs = []
    total = 0
    span = 1
    for _ in range(L):
        span *= b
        offs.append(total)
        total += n_cap // span
    return np.asarray(offs, dtype=np.int64), total


class Tree:
    """Summaries of one (sequence, KV head): level l rows at ``rows[offs[l-1]:]``."""

    def __init__(self, rows: np.ndarray, offs: np.ndarray, b: int, L: int, d: int):
        self.rows = rows
        self.offs = offs
        self.b = b
        self.L = L
        self.d = d

    def level(self, l: int) -> np.ndarray:
        start = int(self.offs[l - 1])
        end = int(self.offs[l]) if l < self.L else self.rows.shape[0]
        return self.rows[start:end]


def build_tree(K, n: int, R, b: int, L: int, store_bf16: bool, n_cap: Optional[int] = None) -> Tree:
    """Build every complete node over the first n keys of one (sequence, KV head)."""
    K = _f32(K)
    R = _f32(R)
    d = K.shape[1]
    n_cap = K.shape[0] if n_cap is None else n_cap
    offs, total = level_row_offsets(n_cap, b, L)
    rows = np.zeros((max(total, 1), d), dtype=np.float32)
    lib().zo_build_tree(_ptr(K, _f32p), n, d, _ptr(R, _f32p), b, L, int(store_bf16),
                        _ptr(rows, _f32p), _ptr(offs, _i64p))
    return Tree(rows, offs, b, L, d)


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------

def cut(z, nodes, p: float):
    """Canonical top-p cut at one level. Returns (kept ascending, T, need, near_tie)."""
    z = _f32(z)
    nodes = np.ascontiguousarray(nodes, dtype=np.int64)
    n = z.shape[0]
    kept = np.empty(max(n, 1), dtype=np.int64)
    T = ctypes.c_uint64(0)
    need = ctypes.c_uint64(0)
    tie = ctypes.c_int(0)
    k = lib().zo_cut(_ptr(z, _f32p), _ptr(nodes, _i64p), n, p_fixed(p), _ptr(kept, _i64p),
                     ctypes.byref(T), ctypes.byref(need), ctypes.byref(tie))
    return kept[:k].copy(), int(T.value), int(need.value), bool(tie.value)


def select(q, tree: Tree, t: int, p: float, cap: Optional[int] = None):
    """Canonical selection for one query head at position t.

    Returns (idx int32 ascending, level_counts int32[L] top level first,
    level_ncand int64[L], near_tie bool)."""
    q = _f32(q)
    if cap is None:
        cap = t + 2
    idx = np.empty(max(cap, 1), dtype=np.int32)
    counts = np.zeros(tree.L, dtype=np.int32)
    ncand = np.zeros(tree.L, dtype=np.int64)
    tie = ctypes.c_int(0)
    n = lib().zo_select(_ptr(q, _f32p), tree.d, _ptr(tree.rows, _f32p), _ptr(tree.offs, _i64p),
                        tree.b, tree.L, t, p_fixed(p), _ptr(idx, _i32p), cap, _ptr(counts, _i32p),
                        _ptr(ncand, _i64p), ctypes.byref(tie))
    return idx[:min(n, cap)].copy(), counts, ncand, bool(tie.value)


def select_f64(q, tree: Tree, t: int, p: float):
    """fp64 rendering of the same traversal. Returns (idx, level_counts, margin)."""
    q = _f32(q)
    cap = t + 2
    idx = np.empty(cap, dtype=np.int32)
    counts = np.zeros(tree.L, dtype=np.int32)
    margin = ctypes.c_double(0.0)
    n = lib().zo_select_f64(_ptr(q, _f32p), tree.d, _ptr(tree.rows, _f32p),
                            _ptr(tree.offs, _i64p), tree.b, tree.L, t, ctypes.c_double(p),
                            _ptr(idx, _i32p), cap, _ptr(counts, _i32p), ctypes.byref(margin))
    return idx[:n].copy(), counts, float(margin.value)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def fp4_round_rows(rows) -> Tuple[np.ndarray, np.ndarray]:
    """Block-scaled 4-bit rounding of [n][d] rows (zo_fp4_round_rows): the
    rounded fp32 values and the per-32-element exponents [n][d / 32]."""
    x = np.ascontiguousarray(rows, dtype=np.float32)
    n, d = x.shape
    assert d % 32 == 0
    out = np.empty_like(x)
    exps = np.empty((n, d // 32), dtype=np.int32)
    lib().zo_fp4_round_rows(_ptr(x, _f32p), n, d, _ptr(out, _f32p), _ptr(exps, _i32p))
    return out, exps


def fp4_tree(tree: "Tree") -> "Tree":
    """The tree with every stored summary row rounded by fp4_round_rows."""
    return Tree(fp4_round_rows(tree.rows)[0], tree.offs, tree.b, tree.L, tree.d)


def attend(q, K, V, idx) -> np.ndarray:
    """fp64 softmax attention of q over rows idx of (K, V)."""
    q = _f32(q)
    K = _f32(K)
    V = _f32(V)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.empty(q.shape[0], dtype=np.float64)
    lib().zo_attend_f64(_ptr(q, _f32p), q.shape[0], _ptr(K, _f32p), _ptr(V, _f32p),
                        _ptr(idx, _i32p), idx.shape[0], _ptr(out, _f64p))
    return out


def dense(q, K, V, t: int) -> np.ndarray:
    return attend(q, K, V, np.arange(t + 1, dtype=np.int32))


# ---------------------------------------------------------------------------
# whole-workload helpers (loops over units and heads; no extra arithmetic)
# ---------------------------------------------------------------------------

def build_trees(K: np.ndarray, seq_len: Sequence[int], R, b: int, L: int, store_bf16: bool,
                units: Optional[List[Tuple[int, int]]] = None):
    """K: [B][Hkv][Ncap][d] fp32 values. Returns {(seq, kvh): Tree}."""
    B, Hkv, n_cap, _ = K.shape
    if units is None:
        units = [(s, h) for s in range(B) for h in range(Hkv)]
    return {(s, h): build_tree(K[s, h], int(seq_len[s]), R, b, L, store_bf16, n_cap)
            for (s, h) in units}


def kv_head(h: int, n_q_heads: int, n_kv_heads: int) -> int:
    return h // (n_q_heads // n_kv_heads)


def p_cover_exact(p: float) -> float:
    """The coverage fraction the fixed-point need actually uses: p_q / 2^32."""
    return p_fixed(p) / 4294967296.0


__all__ = [
    "build", "lib", "exp_c", "round_bf16", "p_fixed", "dot", "score", "build_node",
    "build_node_f64", "level_row_offsets", "Tree", "build_tree", "cut", "select", "select_f64",
    "attend", "dense", "build_trees", "kv_head", "p_cover_exact",
]
