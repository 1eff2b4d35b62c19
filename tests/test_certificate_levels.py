"""How often the tensor-core certificate could hold below the top level (CPU).

The prefill top level is scored on the tensor cores, and a (token, head) row
skips the canonical scores only when the certificate proves that the
canonical cut of every score vector in the box z~ +- delta is one set. This
study asks what the same certificate would give at the lower levels, where
tensor-core scoring of the union of a tile's candidates would apply: for
sampled prefill queries of the c4 recipe (131K context here), the canonical
descent is followed and, at each level, the certificate is evaluated on the
level's frontier with z~ = the scores themselves (no tensor-core error at
all, the most favourable case) and the error bound delta of the tensor-core
scores. The fraction of certified (query, level) cuts is then an upper bound
on what tensor-core scoring below the top level could skip."""
import numpy as np

import oracle
from tree_indexed_sparse_zha_b200 import workloads as W

from test_certificate import certify


def _frontier_scores(q, rows, level, b, inv_sqrt_d):
    """fp32 scores fl(fl(q . s * inv_sqrt_d) + l ln b) of the rows (the dot in
    fp64, rounded once: close to the canonical chain, enough for a study)."""
    dots = (rows.astype(np.float64) @ q.astype(np.float64)).astype(np.float32)
    return (dots * np.float32(inv_sqrt_d) + np.float32(level * np.log(b))).astype(np.float32)


def test_certifiable_fraction_by_level():
    wl = W.make("prefill-deep-1m-chunk4k", n_tokens=131072, chunk=64)
    c = wl.cfg
    b, L, d, p = c.block, c.levels, c.head_dim, c.p
    inv_sqrt_d = float(np.float32(1.0 / np.sqrt(d)))
    n = c.n_tokens
    t = n - 1
    K = wl.K.float().numpy()
    R = wl.R.numpy()
    q_all = wl.queries(0).float().numpy()  # [chunk][Hq][d]
    trees = [oracle.build_tree(K[0, kvh], n, R, b, L, True, c.capacity)
             for kvh in range(c.n_kv_heads)]
    certified = np.zeros(L, dtype=np.int64)
    total = np.zeros(L, dtype=np.int64)
    sizes = np.zeros(L, dtype=np.int64)
    rng = np.random.default_rng(11)
    tokens = rng.choice(c.chunk, 8, replace=False)
    for i in tokens:
        for h in range(c.n_q_heads):
            q = q_all[i, h]
            qn = float(np.linalg.norm(q.astype(np.float64)))
            tree = trees[h // c.group]
            nodes = np.arange((t + 1) // b ** L, dtype=np.int64)
            for level in range(L, 0, -1):
                rows = tree.level(level)[nodes]
                z = _frontier_scores(q, rows, level, b, inv_sqrt_d)
                sn = np.linalg.norm(rows.astype(np.float64), axis=1)
                delta = (12.0 * d * 2.0 ** -24 * inv_sqrt_d * qn * sn
                         + 2.0 ** -21 * (2.0 * np.abs(z.astype(np.float64)) + level * np.log(b) + 1))
                ok, _ = certify(z, delta, p)
                certified[L - level] += int(ok)
                total[L - level] += 1
                sizes[L - level] += len(nodes)
                kept = oracle.cut(z, nodes, p)[0]
                if level > 1:
                    nodes = (kept[:, None] * b + np.arange(b)[None, :]).reshape(-1)
    frac = certified / total
    print("level (top first), mean frontier size, certified fraction:")
    for j in range(L):
        print(f"  L{L - j}: {sizes[j] / total[j]:9.1f}  {frac[j]:.3f}")
    # the top level certifies often (as on the GPU); the large deep frontiers
    # rarely do
    assert frac[0] > 0.3
    assert frac[-1] < frac[0]
