"""Pins of the Quantile Balancing oracle (no GPU): the margin definition
against brute-force re-selection, the bias update against the target count,
the histogram against direct counting and the exact quantile."""
import numpy as np

from oracle import qb_oracle as qb


def _inputs(T, E, seed):
    rng = np.random.default_rng(seed)
    s = rng.random((T, E), dtype=np.float32)  # sigmoid-like scores in (0, 1)
    b = (rng.standard_normal(E) * 0.05).astype(np.float32)
    return s, b


def _selected_by_brute_force(s, b, k):
    """Top-k membership by explicit ranking of fl32(s + b), ties to the lower index."""
    key = (s + b[None, :]).astype(np.float32)
    T, E = key.shape
    out = np.zeros((T, E), dtype=bool)
    for t in range(T):
        ranked = sorted(range(E), key=lambda e: (-float(key[t, e]), e))
        out[t, ranked[:k]] = True
    return out


def test_margin_sign_is_the_selection():
    s, b = _inputs(60, 12, 1)
    m32, m64, sel = qb.qb_margins(s, b, 3)
    assert np.array_equal(sel, _selected_by_brute_force(s, b, 3))
    assert np.array_equal(m64 > 0, sel)
    assert np.array_equal(m32 > 0, sel)


def test_moving_one_bias_by_the_margin_flips_exactly_that_token():
    """b_e - m[t,e] +/- eps puts e just above / below token t's boundary."""
    s, b = _inputs(40, 10, 2)
    k = 3
    _, m64, _ = qb.qb_margins(s, b, k)
    rng = np.random.default_rng(3)
    for _ in range(30):
        t, e = int(rng.integers(40)), int(rng.integers(10))
        for eps, want in ((1e-4, True), (-1e-4, False)):
            b2 = b.copy()
            b2[e] = np.float32(float(b[e]) - m64[t, e] + eps)
            assert _selected_by_brute_force(s, b2, k)[t, e] == want


def test_exact_update_gives_each_expert_its_target_alone():
    """With only b_e moved to b_e - q_e, expert e is chosen by exactly c tokens."""
    T, E, k = 200, 16, 4
    s, b = _inputs(T, E, 4)
    _, m64, _ = qb.qb_margins(s, b, k)
    c = qb.qb_target(T, k, E)
    q = qb.qb_quantile_exact(m64, c)
    for e in range(E):
        b2 = b.copy()
        b2[e] = np.float32(float(b[e]) - q[e])
        assert _selected_by_brute_force(s, b2, k)[:, e].sum() == c


def test_uniform_shift_of_all_biases_keeps_the_margins():
    s, b = _inputs(50, 12, 5)
    _, m_a, _ = qb.qb_margins(s.astype(np.float64), b.astype(np.float64), 3)
    _, m_b, _ = qb.qb_margins(s.astype(np.float64), (b + 0.25).astype(np.float64), 3)
    assert np.allclose(m_a, m_b, atol=1e-6)


def test_histogram_counts_and_quantile_resolution():
    T, E, k, nb, lo, hi = 500, 12, 3, 256, -1.0, 1.0
    s, b = _inputs(T, E, 6)
    r = qb.qb_bias_update(s, b, k, nb, lo, hi)
    counts = r["counts"]
    assert counts.shape == (E, nb) and (counts.sum(axis=1) == T).all()
    # every margin lies in its bin's interval (all margins are inside [lo, hi) here)
    m32, _, _ = qb.qb_margins(s, b, k)
    w = (hi - lo) / nb
    direct = np.zeros_like(counts)
    for e in range(E):
        for t in range(T):
            j = int(np.floor((float(m32[t, e]) - lo) / w))
            direct[e, min(max(j, 0), nb - 1)] += 1
    # fp32 binning may move a margin that sits on a bin edge to its neighbour
    assert np.abs(direct - counts).sum() <= 2
    # q lies in the bin of the c-th margin: within one bin plus half the rank gap
    assert np.all(np.abs(r["q"] - r["q_exact"]) <= w + 0.5 * r["rank_gap"] + 1e-12)


def test_sparse_bins_bound_needs_the_rank_gap():
    """With more bins than margins near the boundary the rank gap dominates,
    and the bound still holds."""
    T, E, k, nb, lo, hi = 300, 8, 2, 8192, -1.0, 1.0
    s, b = _inputs(T, E, 7)
    r = qb.qb_bias_update(s, b, k, nb, lo, hi)
    w = (hi - lo) / nb
    err = np.abs(r["q"] - r["q_exact"])
    assert np.all(err <= w + 0.5 * r["rank_gap"] + 1e-12)
    assert np.any(err > w)  # one bin alone would not bound it
    assert np.allclose(r["bias"], b.astype(np.float64) - r["q"])


def test_histogram_quantile_closed_form():
    """One expert whose margins fill bins evenly: the boundary is exact."""
    nb, lo, hi = 8, 0.0, 8.0
    counts = np.array([[4, 4, 4, 4, 4, 4, 4, 4]])  # 32 margins, 4 per unit bin
    # rank 10 from the top: 8 margins in bins 7, 6; 2 more of bin 5's 4
    assert np.isclose(qb.qb_quantile_from_hist(counts, 10, lo, hi)[0], 5.0 + 1.0 - 2 / 4)
