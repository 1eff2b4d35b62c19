"""Pins for the CPU oracle: each test ties the oracle to something other than
itself (a hand-worked example, a closed form, a textbook special case, brute
force on tiny inputs, invariants). CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from tree_indexed_sparse_zha_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32_EPS = 2.0 ** -23


# ---------------------------------------------------------------------------
# canonical scalar helpers
# ---------------------------------------------------------------------------

def test_exp_c_exact_points():
    assert oracle.exp_c(0.0) == 1.0
    assert oracle.exp_c(-87.5) == 0.0
    assert oracle.exp_c(-1000.0) == 0.0
    # exp(-ln 2 * k) sits on exact powers of two up to a few ulp
    for k in range(1, 40):
        x = float(np.float32(-k * math.log(2.0)))
        assert abs(oracle.exp_c(x) / math.exp(x) - 1.0) < 4 * F32_EPS


def test_exp_c_accuracy_and_monotone():
    xs = np.float32(-np.linspace(0.0, 80.0, 20001))
    vals = np.array([oracle.exp_c(float(x)) for x in xs])
    ref = np.exp(xs.astype(np.float64))
    rel = np.abs(vals / ref - 1.0)
    assert rel.max() < 4 * F32_EPS, rel.max()
    # xs is decreasing, so exp_c must be non-increasing along it
    assert np.all(np.diff(vals) <= 0.0)


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 lies exactly halfway between bf16 neighbours 1 and 1 + 2^-7 -> even (1)
    assert oracle.round_bf16(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6 -> even (1 + 2^-6)
    assert oracle.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert oracle.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -20) == 1.0 + 2.0 ** -7
    assert oracle.round_bf16(-3.0) == -3.0


def test_dot_is_a_sequential_chain():
    # 1 + 1e8 rounds to 1e8 in fp32, so the chain 0 -> 1 -> 1e8 -> 0 ends at 0;
    # any other association (or a fused tree) keeps the 1.
    assert oracle.dot([1.0, 1e8, -1e8], [1.0, 1.0, 1.0]) == 0.0
    assert oracle.dot([1e8, -1e8, 1.0], [1.0, 1.0, 1.0]) == 1.0
    rng = np.random.default_rng(1)
    for d in (64, 128):
        a = rng.standard_normal(d).astype(np.float32)
        x = rng.standard_normal(d).astype(np.float32)
        exact = float(np.dot(a.astype(np.float64), x.astype(np.float64)))
        bound = d * F32_EPS * float(np.abs(a.astype(np.float64) * x).sum())
        assert abs(oracle.dot(a, x) - exact) <= bound


def test_p_fixed():
    assert oracle.p_fixed(1.0) == 2 ** 32
    assert oracle.p_fixed(0.5) == 2 ** 31
    assert oracle.p_fixed(0.95) == 4080218931  # 0.95 * 2^32 = 4080218931.2


# ---------------------------------------------------------------------------
# summaries (closed forms and textbook special cases)
# ---------------------------------------------------------------------------

def test_summary_zero_R_is_mean():
    rng = np.random.default_rng(2)
    for b in (2, 4, 8, 256):
        ch = rng.standard_normal((b, 128)).astype(np.float32)
        s = oracle.build_node(ch, np.zeros((16, 128), np.float32))
        mean = ch.astype(np.float64).mean(0)
        assert np.abs(s - mean).max() <= 4 * b * F32_EPS * np.abs(ch).max()


def test_summary_identical_children_is_the_child():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128).astype(np.float32)
    R = (rng.standard_normal((16, 128)) / math.sqrt(128)).astype(np.float32)
    # exact for b = 2 (x/2 + x/2); partial sums k x / b round for larger b
    assert np.array_equal(oracle.build_node(np.tile(x, (2, 1)), R), x)
    for b in (4, 8, 16):
        s = oracle.build_node(np.tile(x, (b, 1)), R)
        assert np.all(np.abs(s - x) <= b * F32_EPS * np.abs(x))


def test_summary_b2_is_mean_of_sigmoids():
    # b = 2: softmax over two children is the logistic function of the logit
    # difference, so s = (1/16) sum_r [sig_r k_a + (1 - sig_r) k_b].
    rng = np.random.default_rng(4)
    for d in (64, 128):
        for _ in range(5):
            ka = rng.standard_normal(d).astype(np.float32)
            kb = rng.standard_normal(d).astype(np.float32)
            R = (rng.standard_normal((16, d)) * 2.0).astype(np.float32)
            s = oracle.build_node(np.stack([ka, kb]), R)
            delta = (R.astype(np.float64) @ (ka.astype(np.float64) - kb)) / math.sqrt(d)
            sig = 1.0 / (1.0 + np.exp(-delta))
            ref = (sig[:, None] * ka + (1.0 - sig[:, None]) * kb).mean(0)
            assert np.abs(s - ref).max() < 2e-5 * max(1.0, np.abs(ref).max())


def test_summary_b2_ln3_gives_three_quarters():
    # every logit difference ln 3 -> weights 3/4 and 1/4
    d = 4
    ka = np.array([1.0, 2.0, -1.0, 0.5], np.float32)
    kb = np.array([0.0, 2.0, -1.0, 0.5], np.float32)
    R = np.zeros((16, d), np.float32)
    R[:, 0] = 2.0 * math.log(3.0)  # (R . (ka - kb)) / sqrt(4) = ln 3
    s = oracle.build_node(np.stack([ka, kb]), R)
    assert np.allclose(s, 0.75 * ka + 0.25 * kb, rtol=0, atol=1e-6)


def test_summary_matches_fp64_formula():
    # the canonical fp32 rendering stays within rounding of the same formula in fp64
    rng = np.random.default_rng(5)
    for b, d in ((4, 128), (4, 64), (8, 128), (256, 128)):
        ch = rng.standard_normal((b, d)).astype(np.float32)
        R = (rng.standard_normal((16, d)) / math.sqrt(d)).astype(np.float32)
        s = oracle.build_node(ch, R)
        ref = oracle.build_node_f64(ch, R)
        assert np.abs(s - ref).max() < 1e-5 * np.abs(ch).max()
        # bf16 storage is the RNE rounding of the fp32 value
        s16 = oracle.build_node(ch, R, store_bf16=True)
        assert all(oracle.round_bf16(float(a)) == float(c) for a, c in zip(s, s16))


def test_tree_levels_use_stored_children():
    # level 2 must be built from the stored level-1 rows (bf16-rounded in bf16 mode)
    rng = np.random.default_rng(6)
    b, L, d, n = 4, 2, 64, 64
    K = rng.standard_normal((n, d)).astype(np.float32)
    R = (rng.standard_normal((16, d)) / math.sqrt(d)).astype(np.float32)
    tr = oracle.build_tree(K, n, R, b, L, store_bf16=True)
    l1 = tr.level(1)
    for j in range(n // (b * b)):
        node = oracle.build_node(l1[j * b:(j + 1) * b], R, store_bf16=True)
        assert np.array_equal(tr.level(2)[j], node)
    # incomplete nodes are not built
    tr2 = oracle.build_tree(K, 30, R, b, L, store_bf16=True, n_cap=n)
    assert np.array_equal(tr2.level(1)[:7], tr.level(1)[:7])
    assert not tr2.level(1)[7:].any()
    # n = 30: level-2 node 0 (tokens 0..15) is complete, node 1 (16..31) is not
    assert np.array_equal(tr2.level(2)[0], tr.level(2)[0]) and not tr2.level(2)[1:].any()


# ---------------------------------------------------------------------------
# the hand-worked example
# ---------------------------------------------------------------------------

def _hand():
    with open(os.path.join(GOLDEN, "hand16.json")) as f:
        g = json.load(f)
    d = g["d"]
    x = np.asarray(g["x"], np.float32)
    K = np.zeros((16, d), np.float32)
    K[:, 0] = x
    V = np.zeros((16, d), np.float32)
    V[:, 0] = np.arange(16)
    V[:, 1] = 1.0
    return g, K, V


def _arith(expr: str, names: dict) -> float:
    """Value of a fixture's closed form: numbers, the given names, + - * / and
    parentheses only."""
    import ast
    import operator

    ops = {ast.Add: operator.add, ast.Sub: operator.sub, ast.Mult: operator.mul,
           ast.Div: operator.truediv}

    def ev(n):
        if isinstance(n, ast.Expression):
            return ev(n.body)
        if isinstance(n, ast.BinOp) and type(n.op) in ops:
            return ops[type(n.op)](ev(n.left), ev(n.right))
        if isinstance(n, ast.UnaryOp) and isinstance(n.op, ast.USub):
            return -ev(n.operand)
        if isinstance(n, ast.Constant) and isinstance(n.value, (int, float)):
            return float(n.value)
        if isinstance(n, ast.Name) and n.id in names:
            return names[n.id]
        raise ValueError(f"unsupported expression: {expr}")

    return ev(ast.parse(expr, mode="eval"))


def test_hand_example():
    g, K, V = _hand()
    tr = oracle.build_tree(K, 16, np.zeros((16, g["d"]), np.float32), g["b"], g["L"], False)
    for l, means in g["summary_means"].items():
        assert tr.level(int(l))[:, 0].tolist() == means
    q = np.asarray(g["query"], np.float32)
    e2, e4 = math.exp(2.0), math.exp(4.0)
    for case in g["cases"]:
        idx, counts, _, _ = oracle.select(q, tr, g["t"], case["p"])
        assert idx.tolist() == case["S"], case["p"]
        assert counts.tolist() == case["level_counts"], case["p"]
        o = oracle.attend(q, K, V, idx)
        o0 = _arith(case["o0"], {"E2": e2, "E4": e4})
        assert abs(o[0] - o0) < 1e-12 and abs(o[1] - 1.0) < 1e-12


# ---------------------------------------------------------------------------
# the top-p cut: brute force over every subset on tiny candidate sets
# ---------------------------------------------------------------------------

def _brute_cut(z, nodes, p):
    """Minimum-cardinality subset with mass >= p*T (exact exp in fp64); among
    those the largest mass; then the lexicographically smallest node list."""
    zmax = max(z)
    m = [math.exp(v - zmax) for v in z]
    T = sum(m)
    n = len(z)
    target = oracle.p_cover_exact(p) * T
    for k in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), k):
            mass = sum(m[i] for i in sub)
            if mass >= target:
                key = (-mass, sorted(nodes[i] for i in sub))
                if best is None or key < best:
                    best = key
        if best is not None:
            return best[1], target, m
    raise AssertionError


def test_cut_brute_force():
    rng = np.random.default_rng(7)
    checked = 0
    for trial in range(400):
        n = int(rng.integers(1, 11))
        z = (rng.standard_normal(n) * rng.choice([0.1, 1.0, 3.0])).astype(np.float32)
        if trial % 5 == 0 and n > 2:
            z[1] = z[0]  # exact ties
        nodes = rng.permutation(50)[:n].astype(np.int64)
        p = float(rng.choice([0.3, 0.5, 0.8, 0.9, 0.95, 0.99]))
        kept, T, need, _ = oracle.cut(z, nodes, p)
        ref, target, m = _brute_cut([float(v) for v in z], [int(v) for v in nodes], p)
        # skip decisions within rounding of the fp64 brute force
        srt = sorted(m, reverse=True)
        cums = np.cumsum(srt)
        if np.min(np.abs(cums - target)) < 1e-6 * cums[-1]:
            continue
        assert kept.tolist() == ref, (z, nodes, p)
        assert need <= T
        checked += 1
    assert checked > 300


def test_cut_near_tie_flags():
    """The near-tie flag, by hand: a cutoff score within 1e-6 relative of a
    sorted neighbour, or a target mass within 1e-6 T of the prefix mass on
    either side of the cut."""
    nodes = np.arange(3, dtype=np.int64)
    # masses 1, 0.61, 0.61: p = 0.6 keeps two, far from either prefix mass, and
    # the third score sits 1e-7 below the cutoff score
    z = np.array([0.0, -0.5, np.nextafter(np.float32(-0.5), np.float32(-1))], np.float32)
    kept, T, need, tie = oracle.cut(z, nodes, 0.6)
    assert kept.tolist() == [0, 1] and tie
    z[2] = -0.6
    assert oracle.cut(z, nodes, 0.6)[3] is False
    # masses 1 and about 1/3: p = 0.75 puts the target on the first prefix
    # mass (2^40), up to the rounding of -ln 3, with scores far apart
    z2 = np.array([0.0, -np.log(3.0)], np.float32)
    kept, T, need, tie = oracle.cut(z2, nodes[:2], 0.75)
    assert abs(int(need) - 2**40) <= 1e-6 * T and tie
    # p = 0.6: the target is 0.2 T below the first prefix mass, no flag
    assert oracle.cut(z2, nodes[:2], 0.6)[3] is False
    # p = 1 makes no cut, so no mass margin applies
    assert oracle.cut(z2, nodes[:2], 1.0)[3] is False


def test_cut_p_one_keeps_everything():
    z = np.array([0.0, -200.0, -100.0, 1.0], np.float32)  # two masses truncate to 0
    kept, T, need, _ = oracle.cut(z, np.arange(4), 1.0)
    assert kept.tolist() == [0, 1, 2, 3]


def test_cut_uniform_masses_keep_ceil_p_n():
    for n in (1, 3, 7, 16, 64, 1000):
        for p in (0.3, 0.5, 0.95, 0.999):
            z = np.full(n, 1.25, np.float32)
            kept, _, _, _ = oracle.cut(z, np.arange(n)[::-1].copy(), p)
            k = math.ceil(n * oracle.p_cover_exact(p) - 1e-12)
            assert kept.tolist() == list(range(k))


# ---------------------------------------------------------------------------
# whole traversal: independent fp64 brute-force traversal on tiny trees
# ---------------------------------------------------------------------------

def _brute_traverse(q, tr, t, p):
    d, b, L = tr.d, tr.b, tr.L
    bL = b ** L
    T_top = (t + 1) // bL
    if T_top == 0:
        return list(range(t + 1)), [0] * L, math.inf
    cand = list(range(T_top))
    counts = []
    margin = math.inf
    kept = []
    for l in range(L, 0, -1):
        if len(cand) > 13:
            return None, None, 0.0  # too many subsets to enumerate
        rows = tr.level(l).astype(np.float64)
        z = [float(rows[c] @ q.astype(np.float64)) / math.sqrt(d) + l * math.log(b) for c in cand]
        kept, target, m = _brute_cut(z, cand, p)
        srt = np.cumsum(sorted(m, reverse=True))
        margin = min(margin, float(np.min(np.abs(srt - target)) / srt[-1]))
        counts.append(len(kept))
        if l > 1:
            cand = [k * b + c for k in kept for c in range(b)]
    S = set([0]) | {k * b + c for k in kept for c in range(b)} | set(range(bL * T_top, t + 1))
    return sorted(S), counts, margin


def test_traversal_brute_force_tiny_trees():
    rng = np.random.default_rng(8)
    checked = 0
    for trial in range(120):
        d = int(rng.choice([4, 64]))
        b = int(rng.choice([2, 4]))
        L = int(rng.integers(1, 4)) if b == 2 else int(rng.integers(1, 3))
        tops = int(rng.integers(1, 4))
        n = b ** L * tops + int(rng.integers(0, b ** L))
        K = rng.standard_normal((n, d)).astype(np.float32) * 2.0
        R = (rng.standard_normal((16, d)) / math.sqrt(d)).astype(np.float32)
        tr = oracle.build_tree(K, n, R, b, L, store_bf16=bool(trial % 2))
        q = (rng.standard_normal(d) * 3.0).astype(np.float32)
        p = float(rng.choice([0.5, 0.8, 0.95]))
        t = n - 1
        S, counts, margin = _brute_traverse(q, tr, t, p)
        if S is None or margin < 1e-5:
            continue
        idx, oc, _, _ = oracle.select(q, tr, t, p)
        assert idx.tolist() == S
        assert oc.tolist() == counts
        checked += 1
    assert checked >= 20


def test_traversal_zero_query_keeps_lowest_indices():
    rng = np.random.default_rng(9)
    b, L, d = 4, 3, 64
    n = 7 * b ** L + 5
    K = rng.standard_normal((n, d)).astype(np.float32)
    R = (rng.standard_normal((16, d)) / math.sqrt(d)).astype(np.float32)
    tr = oracle.build_tree(K, n, R, b, L, True)
    q = np.zeros(d, np.float32)
    for p in (0.3, 0.7, 0.9):
        pp = oracle.p_cover_exact(p)
        idx, counts, _, _ = oracle.select(q, tr, n - 1, p)
        n_cand = 7
        kept = []
        for i in range(L):
            k = math.ceil(n_cand * pp - 1e-12)
            assert counts[i] == k
            kept = list(range(k)) if i == 0 else [c for c in range(k)]
            n_cand = k * b
        # lowest-index nodes at every level: the kept level-1 nodes are 0..k-1
        exp = sorted(set(range(counts[-1] * b)) | {0} | set(range(7 * b ** L, n)))
        assert idx.tolist() == exp


def test_traversal_tiny_p_is_argmax_descent():
    rng = np.random.default_rng(10)
    b, L, d = 4, 4, 128
    checked = 0
    for trial in range(10):
        n = 5 * b ** L + 17
        K = rng.standard_normal((n, d)).astype(np.float32)
        R = (rng.standard_normal((16, d)) / math.sqrt(d)).astype(np.float32)
        tr = oracle.build_tree(K, n, R, b, L, True)
        q = (rng.standard_normal(d) * 4).astype(np.float32)
        cand = list(range(5))
        ok = True
        for l in range(L, 0, -1):
            z = tr.level(l)[cand].astype(np.float64) @ q / math.sqrt(d)
            srt = np.sort(z)
            if len(z) > 1 and srt[-1] - srt[-2] < 1e-4:
                ok = False
            best = cand[int(np.argmax(z))]
            cand = [best * b + c for c in range(b)]
        if not ok:
            continue
        idx, counts, _, _ = oracle.select(q, tr, n - 1, 1e-9)
        assert counts.tolist() == [1] * L
        exp = sorted({0} | {best * b + c for c in range(b)} | set(range(5 * b ** L, n)))
        assert idx.tolist() == exp
        checked += 1
    assert checked >= 5


def test_budget_adapts_to_how_peaked_the_query_is():
    """The budget is per query (lefilia.fr page, par. 3): the sharper a
    query's estimated mass, the fewer nodes cover p of it. For a fixed
    candidate set, scaling the query by a > 0 multiplies every score
    difference by a, and the share of the mass held by the k best candidates
    can only grow with a (its log-derivative is the tilted mean score of the
    k best minus that of all candidates, never negative), so the top level's
    count never grows with a; queries flagged near-tie at some a > 0 are left
    out. Below
    the top the candidates change with the cut above, so there only the
    overall trend is checked: selections shrink from a flat query (a = 0,
    the ceil(p n) lowest nodes) to a sharp one."""
    rng = np.random.default_rng(13)
    b, L, d, p = 4, 4, 64, 0.95
    n = 16 * b ** L
    K = rng.standard_normal((n, d)).astype(np.float32)
    R = (rng.standard_normal((16, d)) / math.sqrt(d)).astype(np.float32)
    tr = oracle.build_tree(K, n, R, b, L, False)
    scales = (0.0, 2.0, 4.0, 8.0, 16.0, 32.0, 64.0)
    checked = 0
    for _ in range(6):
        u = rng.standard_normal(d)
        u /= np.linalg.norm(u)
        tops, sizes = [], []
        for a in scales:
            idx, counts, _, tie = oracle.select((a * u).astype(np.float32), tr, n - 1, p)
            if tie and a > 0:  # a = 0: exact ties everywhere, settled by the index rule
                break
            tops.append(int(counts[0]))
            sizes.append(len(idx))
        else:
            assert all(x >= y for x, y in zip(tops, tops[1:])), tops
            assert sizes[0] > sizes[3] > sizes[5] > sizes[6], sizes
            assert sizes[6] < sizes[0] // 4, sizes
            checked += 1
    assert checked >= 4


def test_no_complete_top_node_is_dense():
    rng = np.random.default_rng(11)
    K = rng.standard_normal((100, 64)).astype(np.float32)
    R = np.zeros((16, 64), np.float32)
    tr = oracle.build_tree(K, 100, R, 4, 4, False)  # b^L = 256 > 100
    idx, counts, _, _ = oracle.select(rng.standard_normal(64).astype(np.float32), tr, 99, 0.5)
    assert idx.tolist() == list(range(100)) and counts.tolist() == [0] * 4


# ---------------------------------------------------------------------------
# attention: the textbook dense softmax, and p = 1 reproduces it
# ---------------------------------------------------------------------------

def test_attend_matches_numpy_softmax():
    rng = np.random.default_rng(12)
    K = rng.standard_normal((300, 64)).astype(np.float32)
    V = rng.standard_normal((300, 64)).astype(np.float32)
    q = (rng.standard_normal(64) * 2).astype(np.float32)
    idx = np.sort(rng.choice(300, 77, replace=False)).astype(np.int32)
    s = K[idx].astype(np.float64) @ q.astype(np.float64) / 8.0
    w = np.exp(s - s.max())
    ref = (w / w.sum()) @ V[idx].astype(np.float64)
    assert np.abs(oracle.attend(q, K, V, idx) - ref).max() < 1e-12


def test_p_one_reproduces_dense_attention():
    wl = W.make("tiny-f32-1k")
    K = wl.K[0, 0].numpy()
    V = wl.V[0, 0].numpy()
    R = wl.R.numpy()
    cfg = wl.cfg
    tr = oracle.build_tree(K, cfg.n_tokens, R, cfg.block, cfg.levels, False)
    q = wl.queries(0)[0, 0].numpy()
    t = cfg.n_tokens - 1
    idx, counts, _, _ = oracle.select(q, tr, t, 1.0)
    assert idx.tolist() == list(range(t + 1))
    s = K.astype(np.float64) @ q.astype(np.float64) / math.sqrt(cfg.head_dim)
    w = np.exp(s - s.max())
    ref = (w / w.sum()) @ V.astype(np.float64)
    assert np.abs(oracle.attend(q, K, V, idx) - ref).max() < 1e-12


# ---------------------------------------------------------------------------
# invariants and fp64 faithfulness on the synthetic workloads
# ---------------------------------------------------------------------------

def _walk_levels(q, tr, t, p):
    """Compose the traversal from the oracle's per-level primitives and check
    coverage and minimality at every level."""
    b, L = tr.b, tr.L
    T_top = (t + 1) // b ** L
    cand = np.arange(T_top, dtype=np.int64)
    kept = cand
    for l in range(L, 0, -1):
        z = np.array([oracle.score(q, tr.level(l)[c], l, b) for c in cand], np.float32)
        kept, T, need, _ = oracle.cut(z, cand, p)
        zmax = float(z.max())
        M = {int(c): int(oracle.exp_c(float(np.float32(v) - np.float32(zmax))) * 2.0 ** 40)
             for c, v in zip(cand, z)}
        covered = sum(M[int(c)] for c in kept)
        assert covered >= need, "coverage"
        if p < 1.0 and len(kept) > 0:
            assert covered - min(M[int(c)] for c in kept) < need, "minimality"
        assert len(kept) <= len(cand)
        if l > 1:
            cand = (kept[:, None] * b + np.arange(b)).reshape(-1)
    return kept


@pytest.mark.parametrize("name", ["tiny-f32-1k", "decode-deep-32k"])
def test_invariants_and_faithfulness(name):
    wl = W.make(name)
    cfg = wl.cfg
    K = wl.K.float().numpy()
    R = wl.R.numpy()
    q_all = wl.queries(0).float().numpy()
    trees = oracle.build_trees(K, [cfg.n_tokens] * cfg.batch, R, cfg.block, cfg.levels,
                               cfg.dtype == "bf16")
    t = cfg.n_tokens - 1
    b, L = cfg.block, cfg.levels
    bL = b ** L
    T_top = (t + 1) // bL
    flagged = 0
    for s in range(cfg.batch):
        for h in range(cfg.n_q_heads):
            tr = trees[(s, h // cfg.group)]
            q = q_all[s, h]
            idx, counts, ncand, tie = oracle.select(q, tr, t, cfg.p)
            flagged += tie
            S = idx.tolist()
            assert S[0] == 0
            assert all(a < c for a, c in zip(S, S[1:]))
            assert set(range(bL * T_top, t + 1)) <= set(S)
            node0 = counts[-1] > 0 and 1 in S and 2 in S  # node (1,0) kept iff tokens 1..b-1 in S
            assert len(S) == b * counts[-1] + (t + 1 - bL * T_top) + (0 if node0 else 1)
            assert np.all(counts <= ncand)
            if h < 2:  # the per-level walk is slow in Python; spot-check it
                kept = _walk_levels(q, tr, t, cfg.p)
                assert sorted(set((kept[:, None] * b + np.arange(b)).reshape(-1).tolist())
                              | {0} | set(range(bL * T_top, t + 1))) == S
            idx64, counts64, margin = oracle.select_f64(q, tr, t, cfg.p)
            if margin > 1e-4:
                assert idx64.tolist() == S and counts64.tolist() == counts.tolist()
    assert flagged <= cfg.batch * cfg.n_q_heads
