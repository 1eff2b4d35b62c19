"""Shared helpers for the GPU parity tests: run the CUDA path through the C-ABI
binding and the oracle on the same seeded tensors."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import tree_indexed_sparse_zha_b200 as z
from tree_indexed_sparse_zha_b200 import workloads as W

TOL = {"bf16": 2e-2, "f32": 1e-5}


class Gpu:
    """The workload's tensors on cuda:0 plus a built tree."""

    def __init__(self, wl: W.Workload, build: bool = True):
        self.wl = wl
        c = wl.cfg
        self.c = c
        dev = torch.device("cuda:0")
        self.dev = dev
        self.cfg = z.make_config(c.head_dim, c.block, c.levels, c.n_q_heads, c.n_kv_heads,
                                 c.batch, c.capacity, c.torch_dtype)
        self.cache = z.Cache(wl.K.to(dev), wl.V.to(dev), wl.R.to(dev).float().contiguous(),
                             z.alloc_tree(self.cfg, dev), wl.seq_len.to(dev).clone())
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        if build:
            z.zha_build_tree(self.cfg, self.cache)
            torch.cuda.synchronize()

    # -- tree ----------------------------------------------------------------
    def tree_unit(self, seq: int, kvh: int):
        """Summary rows of one unit per level, as float32 numpy arrays."""
        c = self.c
        _, offs = z.zha_tree_layout(self.cfg)
        flat = self.cache.tree
        out = []
        for l in range(1, c.levels + 1):
            rows = c.capacity // c.block ** l
            unit = seq * c.n_kv_heads + kvh
            start = offs[l - 1] + unit * rows * c.head_dim
            out.append(flat[start:start + rows * c.head_dim].float().cpu().numpy()
                       .reshape(rows, c.head_dim))
        return out

    def check_status(self):
        torch.cuda.synchronize()
        st = int(self.status.item())
        assert st == 0, z.status_string(st)

    # -- calls ----------------------------------------------------------------
    def decode(self, q: torch.Tensor, p: float, lists: bool = False):
        """zha_decode; with lists, also the per-head token lists the step's
        attention read (zha_decode_kept_lists on the same workspace)."""
        c = self.c
        out = torch.empty_like(q)
        lc = torch.full((c.batch, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=self.dev)
        ws = self.decode_ws()
        z.zha_decode(self.cfg, self.cache, q, p, out, lc, ws, self.status)
        self.check_status()
        if not lists:
            return out.float().cpu().numpy(), lc.cpu().numpy()
        idx, n_idx = self.kept_lists(ws)
        return out.float().cpu().numpy(), lc.cpu().numpy(), idx, n_idx

    def decode_ws(self) -> torch.Tensor:
        if getattr(self, "_dws", None) is None:
            self._dws = z.alloc_workspace(self.cfg, z.ZHA_OP_DECODE, device=self.dev)
        return self._dws

    def kept_lists(self, ws: torch.Tensor, cap: int = None):
        """Per-head token lists [B][Hq][cap] and lengths [B][Hq] (device) of
        the last decode selection on ws."""
        c = self.c
        cap = cap or int(self.cache.seq_len.max().item()) + 2
        idx = torch.full((c.batch, c.n_q_heads, cap), -7, dtype=torch.int32, device=self.dev)
        n_idx = torch.zeros(c.batch, c.n_q_heads, dtype=torch.int32, device=self.dev)
        z.zha_decode_kept_lists(self.cfg, self.cache, ws, idx, n_idx, self.status)
        self.check_status()
        return idx, n_idx

    def dense(self, q: torch.Tensor):
        out = torch.empty_like(q)
        ws = z.alloc_workspace(self.cfg, z.ZHA_OP_DENSE, device=self.dev)
        z.zha_dense_decode(self.cfg, self.cache, q, out, ws)
        torch.cuda.synchronize()
        return out.float().cpu().numpy()

    def select(self, q: torch.Tensor, q_seq, q_pos, p: float, cap: int):
        c = self.c
        nq = q.shape[0]
        qs = torch.as_tensor(q_seq, dtype=torch.int32, device=self.dev)
        qp = torch.as_tensor(q_pos, dtype=torch.int32, device=self.dev)
        idx = torch.full((nq, c.n_q_heads, cap), -7, dtype=torch.int32, device=self.dev)
        n_idx = torch.zeros(nq, c.n_q_heads, dtype=torch.int32, device=self.dev)
        lc = torch.full((nq, c.n_q_heads, c.levels), -1, dtype=torch.int32, device=self.dev)
        ws = z.alloc_workspace(self.cfg, z.ZHA_OP_SELECT, nq, device=self.dev)
        z.zha_select(self.cfg, self.cache, q, qs, qp, p, idx, n_idx, lc, ws, self.status)
        self.check_status()
        return idx, n_idx, lc, qs

    def attend(self, q, qs, idx, n_idx):
        out = torch.empty_like(q)
        ws = z.alloc_workspace(self.cfg, z.ZHA_OP_ATTEND, q.shape[0], device=self.dev)
        z.zha_attend(self.cfg, self.cache, q, qs, idx, n_idx, out, ws, self.status)
        self.check_status()
        return out.float().cpu().numpy()


class Ref:
    """The oracle's trees for the units a test looks at."""

    def __init__(self, wl: W.Workload, n_tokens: int):
        self.wl = wl
        self.c = wl.cfg
        self.K = wl.K.float().numpy()
        self.V = wl.V.float().numpy()
        self.R = wl.R.numpy()
        self.n = n_tokens
        self._trees = {}

    def tree(self, seq: int, kvh: int) -> oracle.Tree:
        key = (seq, kvh)
        if key not in self._trees:
            c = self.c
            self._trees[key] = oracle.build_tree(self.K[seq, kvh], self.n, self.R, c.block,
                                                 c.levels, c.dtype == "bf16", c.capacity)
        return self._trees[key]

    def select(self, q: np.ndarray, seq: int, h: int, t: int, p: float):
        kvh = h // self.c.group
        return oracle.select(q, self.tree(seq, kvh), t, p)

    def attend(self, q, seq, h, idx):
        kvh = h // self.c.group
        return oracle.attend(q, self.K[seq, kvh], self.V[seq, kvh], idx)


def compare_tree(gpu: Gpu, ref: Ref, seq: int, kvh: int):
    got = gpu.tree_unit(seq, kvh)
    exp = ref.tree(seq, kvh)
    for l in range(1, gpu.c.levels + 1):
        a = got[l - 1]
        b = exp.level(l)
        n = min(a.shape[0], b.shape[0])
        assert np.array_equal(a[:n].view(np.uint32), b[:n].view(np.uint32)), \
            f"level {l}: {int((a[:n] != b[:n]).any(1).sum())} rows differ"
