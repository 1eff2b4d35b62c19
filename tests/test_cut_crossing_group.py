"""Workload property behind the traversal's pass count (CPU, no GPU).

The GPU cut takes a first histogram pass that maps each head's scores linearly
onto 256 buckets over [max(zmin, zmax - 32), zmax]. It finds the bucket where
the mass taken in descending score order reaches the target, and hands that
bucket's members to the head's owner CTA when there are at most 512 of them.
The owner then finishes the cut alone, with no further pass over the frontier.
This test restates that bucket map in numpy, with fp64 masses, over the
oracle's tree of one sequence of the 256K decode workload. It checks that
every level's crossing group of every query head fits the 512-member hand-over,
so that the cut costs one histogram pass and one gather per level. It measures
how often work is done, not what is selected: selection parity is covered by
the oracle pins and the GPU tests."""
import numpy as np

import oracle
from tree_indexed_sparse_zha_b200 import workloads as W

GATHER_CAP = 512
N_BUCKETS = 256


def crossing_group(z: np.ndarray, p: float) -> int:
    """Members of the first pass's crossing bucket for one head's scores z."""
    mx, mn = float(z.max()), float(z.min())
    lo = max(mn, mx - 32.0)
    scale = N_BUCKETS / (mx - lo) if mx > lo else 0.0
    bucket = np.clip(np.floor((z.astype(np.float64) - lo) * scale), 0, N_BUCKETS - 1).astype(int)
    mass = np.exp(z.astype(np.float64) - mx)
    per_bucket = np.bincount(bucket, weights=mass, minlength=N_BUCKETS)
    taken = np.cumsum(per_bucket[::-1])
    beta = N_BUCKETS - 1 - int(np.searchsorted(taken, p * mass.sum()))
    return int((bucket == max(beta, 0)).sum())


def test_crossing_group_examples():
    # one dominant score: its bucket alone reaches the target
    z = np.array([10.0, 0.0, 0.0, 0.0], dtype=np.float32)
    assert crossing_group(z, 0.95) == 1
    # equal scores share one bucket
    assert crossing_group(np.zeros(7, dtype=np.float32), 0.5) == 7


def test_headline_crossing_groups_fit_the_gather():
    wl = W.make("decode-deep-256k-b8", batch=1)
    c = wl.cfg
    t = c.n_tokens - 1
    K = wl.K[0, 0].float().numpy()
    q = wl.queries(0).float().numpy()[0]
    tree = oracle.build_tree(K, t + 1, wl.R.numpy(), c.block, c.levels, True, c.capacity)
    inv = np.float32(1.0 / np.sqrt(c.head_dim))
    worst = {}
    for h in range(c.group):
        nodes = np.arange((t + 1) // c.block ** c.levels)
        for lvl in range(c.levels, 0, -1):
            rows = tree.level(lvl)[nodes].astype(np.float64)
            z = ((rows @ q[h].astype(np.float64)).astype(np.float32) * inv
                 + np.float32(lvl * np.log(c.block))).astype(np.float32)
            g = crossing_group(z, c.p)
            worst[lvl] = max(worst.get(lvl, 0), g)
            assert g <= GATHER_CAP, (h, lvl, g, len(nodes))
            kept, _, _, _ = oracle.cut(z, nodes, c.p)
            if lvl > 1:
                nodes = (kept[:, None] * c.block + np.arange(c.block)[None, :]).ravel()
    print("largest crossing group per level (top first):",
          [worst[lvl] for lvl in range(c.levels, 0, -1)])
