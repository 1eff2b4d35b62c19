"""The block-scaled 4-bit (FP4) router variant on the CPU oracle.

lefilia.fr page, paragraph 4: an FP4 variant of the router was tried. The
oracle's zo_fp4_round_rows rounds every stored summary row to e2m1 values
{0, 0.5, 1, 1.5, 2, 3, 4, 6} with one power-of-two scale per 32 elements,
chosen so the block's largest magnitude fits, exact ties to the even code.

Pins of that rounding: hand-worked rows, a brute-force search over every
code and scale on random and tie-heavy blocks, and its invariances. Then the
drift study: the oracle's traversal on the rounded tree against the
canonical selection of the same queries (recall of the canonical token set,
set sizes, exact softmax mass covered, attention error). The GPU path that
scores 4-bit rows is checked against this rounding and traversal bit for
bit in tests/test_gpu_fp4.py."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tree_indexed_sparse_zha_b200 import workloads as W

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def fp4_tree(tree: oracle.Tree) -> oracle.Tree:
    return oracle.fp4_tree(tree)


def test_fp4_rounding_examples():
    row = np.zeros((1, 32), dtype=np.float32)
    row[0, :6] = [6.0, 2.9, -0.74, 0.25, 1.25, 5.0]
    q, e = oracle.fp4_round_rows(row)
    # amax 6 -> scale 1: 2.9 -> 3, -0.74 -> -0.5, 0.25 (tie 0 / 0.5) -> 0,
    # 1.25 (tie 1 / 1.5) -> 1, 5 (tie 4 / 6) -> 4
    assert q[0, :6].tolist() == [6.0, 3.0, -0.5, 0.0, 1.0, 4.0]
    assert e[0, 0] == 0
    row2 = np.full((1, 32), 0.1, dtype=np.float32)
    row2[0, 0] = 12.0  # scale 2: 0.1 / 2 rounds to 0
    q2, e2 = oracle.fp4_round_rows(row2)
    assert q2[0, :2].tolist() == [12.0, 0.0] and e2[0, 0] == 1
    # 0.75 (tie 0.5 / 1) -> 1, 1.75 (tie 1.5 / 2) -> 2, 2.5 (tie 2 / 3) -> 2,
    # 3.5 (tie 3 / 4) -> 4; amax 6.0000005 needs scale 2: 6.0000005 / 2 -> 3,
    # 1 / 2 = 0.5 exactly, 0.4 / 2 = 0.2 -> 0
    row3 = np.zeros((2, 32), dtype=np.float32)
    row3[0, :5] = [0.75, 1.75, 2.5, 3.5, -6.0]
    row3[1, :3] = [np.nextafter(np.float32(6.0), np.float32(7.0)), 1.0, 0.4]
    q3, e3 = oracle.fp4_round_rows(row3)
    assert q3[0, :5].tolist() == [1.0, 2.0, 2.0, 4.0, -6.0] and e3[0, 0] == 0
    assert q3[1, :3].tolist() == [6.0, 1.0, 0.0] and e3[1, 0] == 1
    # an all-zero block keeps scale 1 and stays zero
    q4, e4 = oracle.fp4_round_rows(np.zeros((1, 32), dtype=np.float32))
    assert not q4.any() and e4[0, 0] == 0


def _brute_force_block(x):
    """Smallest e by scanning, then the nearest of the 8 magnitudes times 2^e
    by exact rational distances, ties to the even code."""
    amax = max(abs(Fraction(float(v))) for v in x)
    e = 0
    if amax > 0:
        e = -160
        while Fraction(6) * Fraction(2) ** e < amax:
            e += 1
    scale = Fraction(2) ** e
    out = []
    for v in x:
        a = abs(Fraction(float(v)))
        best = None
        for k, m in enumerate(E2M1):
            dist = abs(a - Fraction(m) * scale)
            if best is None or dist < best[0] or (dist == best[0] and k % 2 == 0):
                best = (dist, k)
        val = float(Fraction(E2M1[best[1]]) * scale)
        out.append(-val if (v < 0 and val != 0) else val)
    return out, e


def test_fp4_rounding_brute_force():
    rng = np.random.default_rng(5)
    blocks = []
    for k in range(40):  # random magnitudes over a wide exponent range
        blocks.append((rng.standard_normal(32) * 2.0 ** rng.integers(-20, 20)).astype(np.float32))
    for k in range(20):  # exact midpoints and code values at a random scale
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 3.0, 6.0])
        v = rng.choice(mids, 32) * rng.choice([-1.0, 1.0], 32)
        v[0] = 6.0  # fixes the scale at 2^k
        blocks.append((v * 2.0 ** int(rng.integers(-8, 8))).astype(np.float32))
    x = np.stack(blocks)  # one block per row, d = 32
    q, e = oracle.fp4_round_rows(x)
    for i in range(x.shape[0]):
        want, we = _brute_force_block(x[i])
        assert e[i, 0] == we, i
        assert q[i].tolist() == want, i


def test_fp4_rounding_invariances():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    q, e = oracle.fp4_round_rows(x)
    # idempotent; commutes with sign flips and with power-of-two scaling
    q2, _ = oracle.fp4_round_rows(q)
    assert np.array_equal(q, q2)
    assert np.array_equal(oracle.fp4_round_rows(-x)[0], -q)
    q8, e8 = oracle.fp4_round_rows(x * np.float32(8.0))
    assert np.array_equal(q8, q * np.float32(8.0)) and np.array_equal(e8, e + 3)
    # every value is a signed magnitude times its block's power of two, within
    # half of the largest gap (1 at scale 1) of its input
    scale = np.repeat(np.ldexp(1.0, e), 32, axis=1)
    assert np.isin(np.abs(q) / scale, E2M1).all()
    assert (np.abs(q - x) <= scale).all()


def _drift(wl, seqs, heads, t, p):
    c = wl.cfg
    K = wl.K.float().numpy()
    V = wl.V.float().numpy()
    R = wl.R.numpy()
    q = wl.queries(0).float().numpy()
    stats = []
    for s in seqs:
        for kvh in range(c.n_kv_heads):
            tree = oracle.build_tree(K[s, kvh], t + 1, R, c.block, c.levels, True, c.capacity)
            tq = fp4_tree(tree)
            for h in range(kvh * c.group, (kvh + 1) * c.group):
                if h not in heads:
                    continue
                qq = q[s, h]
                sel, _, _, _ = oracle.select(qq, tree, t, p)
                sel4, _, _, _ = oracle.select(qq, tq, t, p)
                logits = (K[s, kvh, :t + 1].astype(np.float64) @ qq.astype(np.float64)) / np.sqrt(c.head_dim)
                w = np.exp(logits - logits.max())
                w /= w.sum()
                exact = oracle.attend(qq, K[s, kvh], V[s, kvh], np.arange(t + 1, dtype=np.int32))
                o = oracle.attend(qq, K[s, kvh], V[s, kvh], sel)
                o4 = oracle.attend(qq, K[s, kvh], V[s, kvh], sel4)
                stats.append({
                    "recall": len(np.intersect1d(sel, sel4)) / len(sel),
                    "size_ratio": len(sel4) / len(sel),
                    "mass": w[sel].sum(), "mass4": w[sel4].sum(),
                    "err": np.abs(o - exact).max(), "err4": np.abs(o4 - exact).max(),
                })
    return stats


@pytest.mark.parametrize("name,n", [("decode-deep-32k", 32768), ("decode-wide-256k-b8", 16384)])
def test_fp4_router_drift(name, n):
    wl = W.make(name, n_tokens=n, steps=0)
    c = wl.cfg
    st = _drift(wl, [0], set(range(c.n_q_heads)), n - 1, 0.95)
    recall = np.array([x["recall"] for x in st])
    mass = np.array([x["mass"] for x in st])
    mass4 = np.array([x["mass4"] for x in st])
    err = np.array([x["err"] for x in st])
    err4 = np.array([x["err4"] for x in st])
    ratio = np.array([x["size_ratio"] for x in st])
    print(f"{name}: recall mean {recall.mean():.4f} min {recall.min():.4f}; size ratio "
          f"{ratio.mean():.3f}; exact mass covered {mass.mean():.4f} (canonical) vs "
          f"{mass4.mean():.4f} (fp4); max |o - exact| {err.max():.4f} vs {err4.max():.4f}")
    # the variant's drift stays small on these inputs
    assert recall.mean() > 0.9 and recall.min() > 0.8
    assert mass4.mean() > mass.mean() - 0.02
    assert err4.max() < max(2 * err.max(), 0.05)
