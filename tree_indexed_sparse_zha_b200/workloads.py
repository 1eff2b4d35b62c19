"""Seeded synthetic workloads for the ZHA hot path.

This module only draws random numbers; it holds none of the method's
arithmetic. Both the CUDA path and the CPU oracle consume the tensors it
produces.

The workloads stand in for the long-context retrieval evaluations the
lefilia.fr page reports (RULER-13 at 256K, paragraph 2): keys are a mixture of
64 Gaussian centres per (sequence, KV head), a few "needle" keys are planted at
seeded positions, and each query head looks for its own needles. None of the
evaluation's items is reproduced; only its shape (needle retrieval in long
contexts) is mirrored.

Recipe (per workload, generator seeded with 20261202 + workload index; the
streams are drawn in this order):
  centres      [B][Hkv][64][d] ~ N(0, 1)
  assignments  [B][Hkv][Ncap]  uniform over the 64 centres
  K            centre[assignment] + 0.5 N(0, 1)
  V            N(0, 1)
  R            [16][d] ~ N(0, 1/d)            (variance 1/d)
  needles      per query head: a count uniform in [lo, hi], positions uniform in
               [1, n) (token 0 is always attended anyway), fresh N(0, 1) keys
               written over K at those positions of the head's KV head
  queries      q = 8 normalize(mean of the head's needle keys) + N(0, 0.3)
               (variance 0.3); decode steps redraw the noise every step
Decode steps append one token per sequence drawn from the same mixture.
Values are drawn in fp32 and rounded to nearest-even bf16 where the workload
is bf16.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, Optional, Tuple

import torch

SEED_BASE = 20261202
N_CENTRES = 64
N_REF = 16


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    index: int            # seed offset
    dtype: str            # "f32" or "bf16"
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_tokens: int         # cache length per sequence before any step / chunk
    block: int
    levels: int
    p: float
    needles: Tuple[int, int]   # inclusive range of needles per query head
    steps: int = 0        # decode steps (one appended token per sequence each)
    chunk: int = 0        # prefill chunk length (queries per head)
    p_sweep: Tuple[float, ...] = ()

    @property
    def capacity(self) -> int:
        return self.n_tokens + self.steps + self.chunk

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def scaled(self, n_tokens: int, **over) -> "WorkloadConfig":
        """Same recipe at another size (for quick parity cases)."""
        return dataclasses.replace(self, n_tokens=n_tokens,
                                   name=f"{self.name}@{n_tokens}", **over)


CONFIGS: Dict[str, WorkloadConfig] = {
    # tiny fp32 case the oracle finishes instantly: 16 top nodes of 64 tokens
    "tiny-f32-1k": WorkloadConfig("tiny-f32-1k", 0, "f32", 1, 1, 1, 64, 1024, 4, 3, 0.95, (2, 2)),
    # deep tree decode, 32K context, 8 top nodes of 4096 tokens
    "decode-deep-32k": WorkloadConfig("decode-deep-32k", 1, "bf16", 1, 16, 2, 128, 32768, 4, 6,
                                      0.95, (1, 1)),
    # headline: deep tree decode at 256K, 8 sequences, 256 incremental steps
    "decode-deep-256k-b8": WorkloadConfig("decode-deep-256k-b8", 2, "bf16", 8, 16, 2, 128, 262144,
                                          4, 6, 0.95, (1, 8), steps=256),
    # wide tree (b=256, one level) at 256K with a p sweep; p=1 must equal dense
    "decode-wide-256k-b8": WorkloadConfig("decode-wide-256k-b8", 3, "bf16", 8, 16, 2, 128, 262144,
                                          256, 1, 0.95, (1, 8), steps=1,
                                          p_sweep=(0.8, 0.9, 0.95, 0.99, 1.0)),
    # chunked prefill: 4096 queries per head appended to a 1M-token cache
    "prefill-deep-1m-chunk4k": WorkloadConfig("prefill-deep-1m-chunk4k", 4, "bf16", 1, 16, 2, 128,
                                              1048576, 4, 6, 0.95, (1, 4), chunk=4096),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


class Workload:
    """Tensors of one workload on one device.

    K, V        [B][Hkv][Ncap][d] in the workload dtype; rows >= n_tokens hold
                the tokens that decode steps / the prefill chunk append
    R           [16][d] fp32
    seq_len     [B] int32, the initial lengths (n_tokens)
    dirs        [B][Hq][d] fp32 unit needle directions (decode) or
                [chunk][Hq][d] (prefill)
    needle_pos  list of LongTensors, one per (row of dirs, head)
    """

    def __init__(self, cfg: WorkloadConfig, device="cpu", seed: Optional[int] = None):
        self.cfg = cfg
        self.device = torch.device(device)
        self.seed = SEED_BASE + cfg.index if seed is None else seed
        g = _gen(self.seed, self.device)
        B, Hkv, Hq, d = cfg.batch, cfg.n_kv_heads, cfg.n_q_heads, cfg.head_dim
        ncap = cfg.capacity
        dev = self.device
        centres = torch.randn(B, Hkv, N_CENTRES, d, generator=g, device=dev)
        assign = torch.randint(0, N_CENTRES, (B, Hkv, ncap), generator=g, device=dev)
        K = torch.gather(centres, 2, assign.unsqueeze(-1).expand(B, Hkv, ncap, d))
        K.add_(torch.randn(B, Hkv, ncap, d, generator=g, device=dev), alpha=0.5)
        del assign
        V = torch.randn(B, Hkv, ncap, d, generator=g, device=dev)
        self.R = torch.randn(N_REF, d, generator=g, device=dev) * (1.0 / d) ** 0.5
        # needles: decode -> one query row per sequence; prefill -> one per chunk token
        n_rows = cfg.chunk if cfg.chunk else B
        lo, hi = cfg.needles
        n = cfg.n_tokens
        counts = torch.randint(lo, hi + 1, (n_rows, Hq), generator=g, device=dev)
        pos = torch.randint(1, n, (n_rows, Hq, hi), generator=g, device=dev)
        keys = torch.randn(n_rows, Hq, hi, d, generator=g, device=dev)
        valid = torch.arange(hi, device=dev) < counts.unsqueeze(-1)
        mean = (keys * valid.unsqueeze(-1)).sum(2) / counts.unsqueeze(-1)
        self.dirs = mean / mean.norm(dim=-1, keepdim=True)
        # plant the needle keys; when two needles hit the same cache row the one
        # with the larger needle id wins (deterministic on every device)
        seq = (torch.zeros(n_rows, dtype=torch.long, device=dev) if cfg.chunk
               else torch.arange(n_rows, device=dev))
        kvh = torch.arange(Hq, device=dev) // cfg.group
        row = ((seq.view(-1, 1, 1) * Hkv + kvh.view(1, -1, 1)) * ncap + pos)[valid]
        nid = torch.arange(n_rows * Hq * hi, device=dev).view(n_rows, Hq, hi)[valid]
        uniq, inv = torch.unique(row, return_inverse=True)
        win = torch.full((uniq.numel(),), -1, dtype=torch.long, device=dev)
        win.scatter_reduce_(0, inv, nid, reduce="amax")
        K.view(-1, d)[uniq] = keys.view(-1, d)[win]
        self.needle_pos = pos
        self.needle_count = counts
        self.K = K.to(cfg.torch_dtype)
        self.V = V.to(cfg.torch_dtype)
        del K, V
        self.seq_len = torch.full((B,), n, dtype=torch.int32, device=dev)
        self._qgen_seed = self.seed * 1000003 + 17

    # -- queries -----------------------------------------------------------
    def queries(self, step: int = 0) -> torch.Tensor:
        """[rows][Hq][d] queries for decode step `step` (or the prefill chunk)."""
        g = _gen(self._qgen_seed + step, self.device)
        noise = torch.randn(self.dirs.shape, generator=g, device=self.device) * (0.3 ** 0.5)
        return (8.0 * self.dirs + noise).to(self.cfg.torch_dtype)

    # -- appended tokens are pre-drawn into the capacity rows -------------
    def step_rows(self, step: int) -> int:
        """Cache row written by decode step `step` (1-based): n_tokens + step - 1."""
        return self.cfg.n_tokens + step - 1


def make(name_or_cfg, device="cpu", n_tokens: Optional[int] = None, **over) -> Workload:
    cfg = CONFIGS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    if n_tokens is not None or over:
        cfg = cfg.scaled(n_tokens if n_tokens is not None else cfg.n_tokens, **over)
    return Workload(cfg, device)
