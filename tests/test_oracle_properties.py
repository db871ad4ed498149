"""Property tests of the CPU oracle on random small cases (hypothesis).

Each property is fixed by the mathematics, not by the oracle's own code:
selection equals sorting by (score descending, index ascending); it is
unchanged by adding a constant or scaling by a positive factor; calibration
counts are bounded by the number of queries times the budget, and for the
full-head plane itself (a plane equal to the full one) they reach the bound.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle.fasa_oracle as O

SETTINGS = settings(max_examples=60, deadline=None)


def _scores(seed, n, ties):
    r = np.random.default_rng(seed)
    s = r.standard_normal(n)
    if ties:  # a few values repeated to force ties
        s = np.round(s * 2) / 2
    return s


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), n=st.integers(1, 80), k=st.integers(1, 100), ties=st.booleans())
def test_select_is_sorted_prefix(seed, n, k, ties):
    s = _scores(seed, n, ties)
    want = sorted(range(n), key=lambda t: (-s[t], t))[:min(k, n)]
    assert list(O.select_critical_set(s, k)) == sorted(want)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), n=st.integers(1, 60), k=st.integers(1, 60),
       shift=st.integers(-8, 8), scale=st.sampled_from([0.25, 0.5, 2.0, 4.0]))
def test_select_invariant_under_exact_monotone_maps(seed, n, k, shift, scale):
    # dyadic values, so shifting and scaling by powers of two stay exact
    s = np.round(_scores(seed, n, False) * 64) / 64
    a = O.select_critical_set(s, k)
    b = O.select_critical_set(s * scale + shift, k)
    assert np.array_equal(a, b)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), W=st.integers(1, 3), L=st.integers(1, 40), K=st.integers(1, 50))
def test_calibration_counts_bounds(seed, W, L, K):
    r = np.random.default_rng(seed)
    planes = r.standard_normal((W, 65, L)).astype(np.float32)
    planes[:, 7] = planes[:, 64]            # FC 7 carries the full head exactly
    c = O.calibration_counts(planes, K)
    keff = min(K, L)
    assert c.min() >= 0 and c.max() <= W * keff
    assert c[7] == W * keff
    d = O.dominant_from_counts(c, 5)
    assert d[0] == 7 or c[d[0]] == W * keff   # a maximal count comes first (ties to the lower FC)
    assert list(d) == sorted(d, key=lambda i: (-c[i], i))


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), G=st.integers(1, 4), L=st.integers(1, 30), pos=st.integers(0, 5000))
def test_tip_all_fcs_is_group_dot_product(seed, G, L, pos):
    r = np.random.default_rng(seed)
    q = r.standard_normal((G, 128))
    k = r.standard_normal((L, 128))
    qr = O.rotate_queries(q.astype(np.float32), pos, 1e4)
    allfc = np.arange(64)
    s = O.tip_scores(qr, O.sketch_rows(k, allfc), allfc)
    want = (qr.sum(0)[None, :] * k).sum(1)
    assert np.allclose(s, want, rtol=1e-12, atol=1e-12 * (np.abs(qr).sum() * np.abs(k).max() + 1))
