"""Pins of the hybrid-clustering oracle (HyperVAttention §4.2, Eq. (6);
readings C15-C19 in oracle/cluster_oracle.py): hand-worked ratios and a
hand-worked intermediate update, scipy's nearest-centroid assignment for a
whole-sequence update, and the invariants of Eq. (6) and of the subset."""
import math

import numpy as np
import pytest
from scipy.cluster.vq import vq

import oracle as orc


def test_lowe_ratio_hand_worked():
    # 1 x 1 x 3 lattice, one token per cell, windows of 3 cells along w (clipped)
    x = np.array([[0.0], [1.0], [3.0]])
    mu = np.array([[0.5], [2.0], [2.5]])
    rho = orc.lowe_ratio(x, mu, (1, 1, 3), (1, 1, 1), (1, 1, 3))
    # token 0: cells {0, 1}: d = 0.5, 2 -> 0.25; token 1: cells {0, 1, 2}: d = 0.5, 1, 1.5 -> 0.5;
    # token 2: cells {1, 2}: d = 1, 0.5 -> 0.5
    assert np.allclose(rho, [0.25, 0.5, 0.5], rtol=0, atol=1e-15)
    # a tie at the cut goes to the lower token index
    assert orc.ambiguous_subset(rho, 1 / 3).tolist() == [1]
    assert orc.ambiguous_subset(rho, 0.5).tolist() == [1, 2]


def test_lowe_ratio_single_centroid_window_and_equidistant_token():
    x = np.array([[0.0], [5.0]])
    rho = orc.lowe_ratio(x, x.copy(), (1, 1, 2), (1, 1, 1), (1, 1, 1))
    assert rho.tolist() == [0.0, 0.0]
    # a token halfway between two centroids: d1 = d2
    rho = orc.lowe_ratio(np.array([[1.0], [2.0]]), np.array([[0.0], [2.0]]), (1, 1, 2), (1, 1, 1), (1, 1, 2))
    assert rho[0] == 1.0 and rho[1] == 0.0


@pytest.mark.parametrize("seed", [0, 1])
def test_ratio_and_subset_invariants(seed):
    rng = np.random.default_rng(seed)
    grid, cell, window = (4, 6, 6), (2, 2, 3), (3, 3, 3)
    x = rng.standard_normal((int(np.prod(grid)), 8))
    a, mu, rho, sub = orc.hybrid_anchor(x, grid, cell, window, 3, 0.15)
    assert np.all((rho >= 0) & (rho <= 1))
    assert sub.size == math.ceil(0.15 * x.shape[0])
    assert np.all(np.diff(sub) > 0)
    rest = np.setdiff1d(np.arange(x.shape[0]), sub)
    assert rho[sub].min() >= rho[rest].max()
    # the anchor's clusters are the plain local-window clustering
    a2, mu2 = orc.local_window_clustering(x, grid, cell, window, 3)
    assert np.array_equal(a, a2) and np.array_equal(mu, mu2)
    # d1 belongs to the token's last assignment: rho computed by brute force for a few tokens
    _, mu_last = orc.local_window_clustering(x, grid, cell, window, 2)
    counts = orc.cell_counts(grid, cell)
    g = orc.token_cells(grid, cell)
    for l in rng.choice(x.shape[0], size=10, replace=False):
        u = g[l]
        cand = orc.window_cells((u // (counts[1] * counts[2]), (u // counts[2]) % counts[1], u % counts[2]),
                                counts, window)
        d = np.sort(np.linalg.norm(mu_last[cand] - x[l], axis=1))
        assert abs(rho[l] - d[0] / d[1]) < 1e-12
        assert cand[np.argmin(np.linalg.norm(mu_last[cand] - x[l], axis=1))] == a[l]


def test_hybrid_update_hand_worked():
    a_prev = np.array([0, 0, 1])
    mu_prev = np.array([[0.0], [10.0]])
    x_new = np.array([[0.0], [9.0], [10.0]])
    a, mu, changed = orc.hybrid_update(x_new, a_prev, mu_prev, np.array([1]))
    assert a.tolist() == [0, 1, 1] and changed.tolist() == [0, 1]
    assert mu[:, 0].tolist() == [0.0, 9.5]
    # a token outside the subset keeps its cluster even when another centroid is nearer
    a, mu, changed = orc.hybrid_update(np.array([[9.0], [9.0], [10.0]]), a_prev, mu_prev, np.array([1]))
    assert a.tolist() == [0, 1, 1] and mu[0, 0] == 9.0 and mu[1, 0] == 9.5


def test_hybrid_update_empty_subset_is_identity():
    rng = np.random.default_rng(3)
    x, mu = rng.standard_normal((50, 4)), rng.standard_normal((6, 4))
    a_prev = rng.integers(0, 6, size=50)
    a, mu2, changed = orc.hybrid_update(x, a_prev, mu, np.zeros(0, dtype=np.int64))
    assert np.array_equal(a, a_prev) and np.array_equal(mu2, mu) and changed.size == 0


def test_hybrid_update_whole_sequence_is_nearest_centroid_then_means_of_changed():
    rng = np.random.default_rng(4)
    x, mu = rng.standard_normal((300, 5)), rng.standard_normal((12, 5))
    a_prev = rng.integers(0, 12, size=300)
    a, mu2, changed = orc.hybrid_update(x, a_prev, mu, np.arange(300))
    want, _ = vq(x, mu)
    assert np.array_equal(a, want)
    for u in range(12):
        if u in set(changed.tolist()) and np.any(a == u):
            assert np.allclose(mu2[u], x[a == u].mean(axis=0), rtol=0, atol=1e-12)
        else:
            assert np.array_equal(mu2[u], mu[u])
    moved = a != a_prev
    assert set(changed.tolist()) == set(a_prev[moved].tolist()) | set(a[moved].tolist())
