"""B200-native hot path of Zyphra Hierarchical Attention (ZHA).

Thin ctypes binding over ``libzha.so`` (sm_100a CUDA kernels behind the C-ABI
declared in ``include/zha.h``). The functions keep the C names and only
marshal arguments: every step of the path runs in the library's kernels on the
caller's current CUDA stream. PyTorch provides device memory and streams.

If the library is missing or cannot be loaded, importing the binding's
functions raises immediately: there is no CPU or eager fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzha.so")

ZHA_OK = 0
ZHA_ERR_INVALID_ARG = 1
ZHA_ERR_UNSUPPORTED = 2
ZHA_ERR_CUDA = 4
ZHA_ERR_CAPACITY = 8
ZHA_ERR_WORKSPACE = 16
ZHA_ERR_TIMEOUT = 32
ZHA_ERR_INTERNAL = 64

ZHA_F32 = 0
ZHA_BF16 = 1

ZHA_OP_SELECT = 0
ZHA_OP_ATTEND = 1
ZHA_OP_DECODE = 2
ZHA_OP_PREFILL = 3
ZHA_OP_DENSE = 4

EXPORTS = (
    "zha_status_string", "zha_tree_layout", "zha_workspace_bytes", "zha_build_tree",
    "zha_extend_tree", "zha_select", "zha_attend", "zha_decode", "zha_decode_select",
    "zha_decode_attend", "zha_decode_stats", "zha_prefill_chunk", "zha_dense_decode",
    "zha_decode_noalloc", "zha_prefill_top_scores", "zha_decode_kept_lists",
    "zha_fp4_tree_bytes", "zha_fp4_quantize_tree", "zha_decode_fp4",
)


class zha_config(ctypes.Structure):
    _fields_ = [
        ("head_dim", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("levels", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class zha_cache(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("r", ctypes.c_void_p),
        ("tree", ctypes.c_void_p),
        ("seq_len", ctypes.c_void_p),
    ]


class ZhaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libzha.so (built in-tree by ``__graft_entry__.build()``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libzha.so not found at {LIB_PATH}; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        c_cfg, c_cache = P(zha_config), P(zha_cache)
        vp, i32, i64, d, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double,
                               ctypes.c_size_t)
        sig = {
            "zha_status_string": ([i32], ctypes.c_char_p),
            "zha_tree_layout": ([c_cfg, P(sz), P(i64)], i32),
            "zha_workspace_bytes": ([c_cfg, i32, i64, P(sz)], i32),
            "zha_build_tree": ([c_cfg, c_cache, vp], i32),
            "zha_extend_tree": ([c_cfg, c_cache, vp, i64, vp], i32),
            "zha_select": ([c_cfg, c_cache, vp, vp, vp, i64, d, vp, i64, vp, vp, vp, sz, vp, vp],
                           i32),
            "zha_attend": ([c_cfg, c_cache, vp, vp, i64, vp, i64, vp, vp, vp, sz, vp, vp], i32),
            "zha_decode": ([c_cfg, c_cache, vp, d, vp, vp, vp, sz, vp, vp], i32),
            "zha_decode_select": ([c_cfg, c_cache, vp, d, vp, vp, sz, vp, vp], i32),
            "zha_decode_attend": ([c_cfg, c_cache, vp, vp, vp, sz, vp], i32),
            "zha_decode_stats": ([c_cfg, vp, sz, vp, vp], i32),
            "zha_prefill_chunk": ([c_cfg, c_cache, vp, i32, i64, i64, d, vp, vp, vp, sz, vp, vp],
                                  i32),
            "zha_dense_decode": ([c_cfg, c_cache, vp, vp, vp, sz, vp], i32),
            "zha_decode_noalloc": ([c_cfg, c_cache, vp, d, vp, vp, vp, vp], i32),
            "zha_decode_kept_lists": ([c_cfg, c_cache, vp, sz, vp, i64, vp, vp, vp], i32),
            "zha_fp4_tree_bytes": ([c_cfg, P(sz)], i32),
            "zha_fp4_quantize_tree": ([c_cfg, c_cache, vp, vp, vp], i32),
            "zha_decode_fp4": ([c_cfg, c_cache, vp, vp, d, vp, vp, vp, sz, vp, vp], i32),
            "zha_prefill_top_scores": ([c_cfg, c_cache, vp, i32, i64, i64, d, vp, vp, vp, sz, vp,
                                        vp], i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().zha_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != ZHA_OK:
        raise ZhaError(fn, status)


def _device_tensor(t: torch.Tensor, what: str = "tensor") -> torch.Tensor:
    """Every pointer the library takes is memory of the current CUDA device,
    read or written by its kernels: a host tensor, or one on another device, is
    refused here, before any launch."""
    if not t.is_cuda:
        raise ValueError(f"libzha takes CUDA device tensors; {what} is on {t.device}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"libzha launches on the current device "
                         f"(cuda:{torch.cuda.current_device()}); {what} is on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"libzha needs contiguous tensors; {what} is not")
    return t


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(_device_tensor(t).data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---------------------------------------------------------------------------
# configuration / cache handles
# ---------------------------------------------------------------------------

@dataclass
class Cache:
    """Device tensors one call works on (all caller-owned)."""
    k: torch.Tensor           # [B][Hkv][Ncap][d]
    v: torch.Tensor
    r: torch.Tensor           # [16][d] fp32
    tree: torch.Tensor        # flat buffer of zha_tree_layout() bytes (any dtype view)
    seq_len: torch.Tensor     # [B] int32

    def c(self) -> zha_cache:
        for name in ("k", "v", "r", "tree", "seq_len"):
            _device_tensor(getattr(self, name), f"cache.{name}")
        return zha_cache(self.k.data_ptr(), self.v.data_ptr(), self.r.data_ptr(),
                         self.tree.data_ptr(), self.seq_len.data_ptr())


def make_config(head_dim: int, block: int, levels: int, n_q_heads: int, n_kv_heads: int,
                batch: int, capacity: int, dtype: torch.dtype) -> zha_config:
    return zha_config(head_dim, block, levels, n_q_heads, n_kv_heads, batch, capacity,
                      ZHA_BF16 if dtype == torch.bfloat16 else ZHA_F32, 0)


def zha_tree_layout(cfg: zha_config):
    nbytes = ctypes.c_size_t(0)
    offs = (ctypes.c_int64 * max(cfg.levels, 1))()
    _check("zha_tree_layout", lib().zha_tree_layout(ctypes.byref(cfg), ctypes.byref(nbytes), offs))
    return nbytes.value, [offs[i] for i in range(cfg.levels)]


def zha_workspace_bytes(cfg: zha_config, op: int, max_queries: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check("zha_workspace_bytes",
           lib().zha_workspace_bytes(ctypes.byref(cfg), op, max_queries, ctypes.byref(n)))
    return n.value


def alloc_tree(cfg: zha_config, device="cuda") -> torch.Tensor:
    nbytes, _ = zha_tree_layout(cfg)
    dt = torch.bfloat16 if cfg.dtype == ZHA_BF16 else torch.float32
    return torch.zeros(max(nbytes // dt.itemsize, 1), dtype=dt, device=device)


def zha_fp4_tree_bytes(cfg: zha_config) -> int:
    n = ctypes.c_size_t(0)
    _check("zha_fp4_tree_bytes", lib().zha_fp4_tree_bytes(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def alloc_fp4_tree(cfg: zha_config, device="cuda") -> torch.Tensor:
    return torch.zeros(zha_fp4_tree_bytes(cfg), dtype=torch.uint8, device=device)


def alloc_workspace(cfg: zha_config, op: int, max_queries: int = 0, device="cuda") -> torch.Tensor:
    return torch.empty(zha_workspace_bytes(cfg, op, max_queries), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# entry points (same names as the C-ABI)
# ---------------------------------------------------------------------------

def zha_build_tree(cfg: zha_config, cache: Cache, stream=None):
    c = cache.c()
    _check("zha_build_tree", lib().zha_build_tree(ctypes.byref(cfg), ctypes.byref(c),
                                                  _stream(stream)))


def zha_extend_tree(cfg: zha_config, cache: Cache, old_len: torch.Tensor, max_new_tokens: int,
                    stream=None):
    c = cache.c()
    _check("zha_extend_tree", lib().zha_extend_tree(ctypes.byref(cfg), ctypes.byref(c),
                                                    _ptr(old_len), max_new_tokens,
                                                    _stream(stream)))


def zha_select(cfg: zha_config, cache: Cache, q: torch.Tensor, q_seq: torch.Tensor,
               q_pos: torch.Tensor, p: float, idx: torch.Tensor, n_idx: torch.Tensor,
               level_counts: Optional[torch.Tensor], ws: torch.Tensor,
               dev_status: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    nq = q.shape[0]
    _check("zha_select", lib().zha_select(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), _ptr(q_seq), _ptr(q_pos), nq, float(p),
        _ptr(idx), idx.shape[-1], _ptr(n_idx), _ptr(level_counts), _ptr(ws), ws.numel(),
        _ptr(dev_status), _stream(stream)))


def zha_attend(cfg: zha_config, cache: Cache, q: torch.Tensor, q_seq: torch.Tensor,
               idx: torch.Tensor, n_idx: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
               dev_status: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    _check("zha_attend", lib().zha_attend(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), _ptr(q_seq), q.shape[0], _ptr(idx),
        idx.shape[-1], _ptr(n_idx), _ptr(out), _ptr(ws), ws.numel(), _ptr(dev_status),
        _stream(stream)))


def zha_decode(cfg: zha_config, cache: Cache, q: torch.Tensor, p: float, out: torch.Tensor,
               level_counts: Optional[torch.Tensor], ws: torch.Tensor,
               dev_status: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    _check("zha_decode", lib().zha_decode(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), float(p), _ptr(out), _ptr(level_counts),
        _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))


def zha_fp4_quantize_tree(cfg: zha_config, cache: Cache, fp4_tree: torch.Tensor,
                          old_len: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    _check("zha_fp4_quantize_tree", lib().zha_fp4_quantize_tree(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(fp4_tree), _ptr(old_len), _stream(stream)))


def zha_decode_fp4(cfg: zha_config, cache: Cache, fp4_tree: torch.Tensor, q: torch.Tensor,
                   p: float, out: torch.Tensor, level_counts: Optional[torch.Tensor],
                   ws: torch.Tensor, dev_status: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    _check("zha_decode_fp4", lib().zha_decode_fp4(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(fp4_tree), _ptr(q), float(p), _ptr(out),
        _ptr(level_counts), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))


def zha_decode_select(cfg: zha_config, cache: Cache, q: torch.Tensor, p: float,
                      level_counts: Optional[torch.Tensor], ws: torch.Tensor,
                      dev_status: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    _check("zha_decode_select", lib().zha_decode_select(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), float(p), _ptr(level_counts), _ptr(ws),
        ws.numel(), _ptr(dev_status), _stream(stream)))


def zha_decode_attend(cfg: zha_config, cache: Cache, q: torch.Tensor, out: torch.Tensor,
                      ws: torch.Tensor, stream=None):
    c = cache.c()
    _check("zha_decode_attend", lib().zha_decode_attend(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), _ptr(out), _ptr(ws), ws.numel(),
        _stream(stream)))


def zha_decode_stats(cfg: zha_config, ws: torch.Tensor, stats: torch.Tensor, stream=None):
    _check("zha_decode_stats", lib().zha_decode_stats(
        ctypes.byref(cfg), _ptr(ws), ws.numel(), _ptr(stats), _stream(stream)))


def zha_decode_kept_lists(cfg: zha_config, cache: Cache, ws: torch.Tensor, idx: torch.Tensor,
                          n_idx: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
                          stream=None):
    """Per-head token lists ([B][Hq][idx_cap] int32, lengths [B][Hq]) of the
    last decode selection left in ws."""
    c = cache.c()
    _check("zha_decode_kept_lists", lib().zha_decode_kept_lists(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(ws), ws.numel(), _ptr(idx), idx.shape[-1],
        _ptr(n_idx), _ptr(dev_status), _stream(stream)))


def zha_prefill_chunk(cfg: zha_config, cache: Cache, q: torch.Tensor, seq: int, chunk_start: int,
                      p: float, out: torch.Tensor, level_counts: Optional[torch.Tensor],
                      ws: torch.Tensor, dev_status: Optional[torch.Tensor] = None, stream=None):
    c = cache.c()
    _check("zha_prefill_chunk", lib().zha_prefill_chunk(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), seq, chunk_start, q.shape[0], float(p),
        _ptr(out), _ptr(level_counts), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))


def zha_dense_decode(cfg: zha_config, cache: Cache, q: torch.Tensor, out: torch.Tensor,
                     ws: torch.Tensor, stream=None):
    c = cache.c()
    _check("zha_dense_decode", lib().zha_dense_decode(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), _ptr(out), _ptr(ws), ws.numel(),
        _stream(stream)))


def zha_prefill_top_scores(cfg: zha_config, cache: Cache, q: torch.Tensor, seq: int,
                           chunk_start: int, p: float, z_top: Optional[torch.Tensor],
                           certified: Optional[torch.Tensor], ws: torch.Tensor,
                           dev_status: Optional[torch.Tensor] = None, stream=None):
    """Tensor-core top-level scores (z_top [T][Hq][capacity // b**L] fp32) and
    per-(token, head) certificates (certified [T][Hq] int32) of a prefill chunk
    whose tree is already built."""
    c = cache.c()
    _check("zha_prefill_top_scores", lib().zha_prefill_top_scores(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), seq, chunk_start, q.shape[0], float(p),
        _ptr(z_top), _ptr(certified), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))


def zha_decode_noalloc(cfg: zha_config, cache: Cache, q: torch.Tensor, p: float,
                       out: torch.Tensor, level_counts: Optional[torch.Tensor],
                       dev_status: Optional[torch.Tensor] = None, stream=None):
    """zha_decode with the library's static 64 MiB device scratch as workspace
    (no allocation). Calls whose executions overlap share that scratch and race;
    order them on one stream."""
    c = cache.c()
    _check("zha_decode_noalloc", lib().zha_decode_noalloc(
        ctypes.byref(cfg), ctypes.byref(c), _ptr(q), float(p), _ptr(out), _ptr(level_counts),
        _ptr(dev_status), _stream(stream)))


__all__ = [n for n in globals() if n.startswith("zha_")] + [
    "lib", "Cache", "make_config", "alloc_tree", "alloc_fp4_tree", "alloc_workspace", "ZhaError",
    "EXPORTS",
]
