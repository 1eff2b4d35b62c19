"""Soundness of the prefill top-level certificate, on the CPU.

The tensor-core top level keeps exact selections by proof: for a row of
approximate scores z~ with per-node error bounds delta, it picks a candidate set
K and certifies that the canonical cut (the oracle's fixed-point top-p cut)
selects exactly K for every score vector in the box z~ +- delta. The three
conditions (separation, cover, minimality) are restated here from their
derivation, and the claim is checked against the oracle's own cut on many
vectors of the box, its corners included. A wrong direction in any bound (a mass
bound taken from the wrong end of the box, a missing truncation term, a flipped
inequality) certifies some row whose box contains a vector with another cut."""
import numpy as np
import pytest

import oracle

ETA = 2.0 ** -20          # relative error bound of exp_c
TWO40 = 2.0 ** -40


def order_key(z32):
    u = z32.view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def candidate_set(zt, p):
    """Top nodes by z~ whose fp32 softmax mass first reaches p (any choice is
    allowed; the certificate decides whether it is the canonical one)."""
    pr = oracle.p_fixed(p) / 2.0 ** 32
    w = np.exp((zt - zt.max()).astype(np.float32)).astype(np.float32)
    target = np.float32(pr) * w.sum(dtype=np.float32)
    keys = order_key(zt)
    tau = 0
    for bit in range(31, -1, -1):
        cand = tau | (1 << bit)
        if w[keys >= cand].sum(dtype=np.float32) >= target:
            tau = cand
    return keys >= tau


def certify(zt, dl, p):
    """The certificate's three conditions over the box [z~ - delta, z~ + delta]."""
    pq = oracle.p_fixed(p)
    K = candidate_set(zt, p)
    if pq >= 2 ** 32:
        return True, np.ones_like(K)
    pr = pq / 2.0 ** 32
    a = zt.astype(np.float64) - dl
    b = zt.astype(np.float64) + dl
    zr = b.max()
    x = 2.0 ** -24 * (zr - a)
    lo = (1 - ETA) * (1 - x)
    hi = (1 + ETA) * (1 + x + x * x)
    ea = np.exp(a - zr) * lo
    eb = np.exp(b - zr) * hi
    k = int(K.sum())
    r = len(zt) - k
    sep = r == 0 or a[K].min() > b[~K].max()
    s_ka, s_kb, s_rb, s_ra = ea[K].sum(), eb[K].sum(), eb[~K].sum(), ea[~K].sum()
    m_ka = ea[K].min()
    ha = (1 - pr) * s_ka - pr * s_rb
    cover = r == 0 or ha - 2.0 ** -36 * ((1 - pr) * s_ka + pr * s_rb) >= (1 + (1 - pr) * k) * TWO40
    hb = (1 - pr) * s_kb - m_ka - pr * s_ra
    minimal = hb + 2.0 ** -36 * ((1 - pr) * s_kb + m_ka + pr * s_ra) <= -(1 + pr * r) * TWO40
    return bool(sep and cover and minimal), K


def inside(v, lo, hi):
    """fp32 values of v, moved inward until they lie in [lo, hi]."""
    f = v.astype(np.float32)
    f = np.where(f.astype(np.float64) < lo, np.nextafter(f, np.float32(np.inf)), f)
    f = np.where(f.astype(np.float64) > hi, np.nextafter(f, np.float32(-np.inf)), f)
    return f


def box_vectors(zt, dl, K, rng, n_random):
    a = zt.astype(np.float64) - dl
    b = zt.astype(np.float64) + dl
    corners = [
        np.where(K, a, b),   # the members low, the rest high (hardest for cover)
        np.where(K, b, a),   # the members high, the rest low (hardest for minimality)
        a, b, zt.astype(np.float64),
    ]
    out = [inside(c, a, b) for c in corners]
    for _ in range(n_random):
        out.append(inside(rng.uniform(a, b), a, b))
    return out


@pytest.mark.parametrize("p", [0.5, 0.9, 0.95])
def test_certified_rows_have_the_certified_cut(p):
    rng = np.random.default_rng(int(p * 1000))
    certified = rejected = 0
    for trial in range(150):
        n = int(rng.integers(2, 40))
        zt = (rng.normal(0.0, 2.0, n) + rng.normal(0.0, 0.5)).astype(np.float32)
        if trial % 5 == 0:  # near ties around the cut
            zt[rng.integers(0, n)] = zt[rng.integers(0, n)] + np.float32(rng.normal(0, 1e-3))
        dl = rng.uniform(1e-5, 3e-2, n)
        ok, K = certify(zt, dl, p)
        if not ok:
            rejected += 1
            continue
        certified += 1
        expect = np.flatnonzero(K)
        nodes = np.arange(n, dtype=np.int64)
        for z in box_vectors(zt, dl, K, rng, 40):
            kept, _, _, _ = oracle.cut(z, nodes, p)
            assert np.array_equal(kept, expect), (trial, p, z, zt, dl)
    # neither vacuous nor trivially permissive
    assert certified >= 30 and rejected >= 5, (certified, rejected)


def test_keep_all_is_always_certified():
    zt = np.array([0.3, -1.0, 2.0], dtype=np.float32)
    ok, K = certify(zt, np.full(3, 0.5), 1.0)
    assert ok and K.all()


def test_a_box_straddling_the_cut_is_rejected():
    # two equal best scores with p just above one node's share: the cut needs
    # one of them, and which one depends on their order inside the box
    zt = np.array([1.0, 1.0, -5.0], dtype=np.float32)
    ok, _ = certify(zt, np.full(3, 1e-3), 0.4)
    assert not ok
