"""Pins of the clustering oracle (HyperVAttention §2 Eq. (1), (4), §4.1 Eq. (5))
against hand-worked cases, a library k-means step, invariants and the
unpermuted path.  CPU only."""
import dataclasses

import numpy as np
import pytest
from scipy.cluster.vq import vq

import oracle as orc
from video_inputs import WORKLOADS, make_qkv



def _hand(x, n_iter=1):
    return orc.local_window_clustering(np.array(x, dtype=np.float64)[:, None], (1, 1, 6), (1, 1, 2), (1, 1, 3), n_iter)


@pytest.mark.parametrize("x,assign,mu", [
    ([0, 4, 5, 6, 10, 11], [0, 1, 1, 1, 2, 2], [0, 5, 10.5]),          # case A: a token moves to the next cell
    ([0, 2.5, 5, 6, 10, 11], [0, 0, 1, 1, 2, 2], [1.25, 5.5, 10.5]),    # case B: tie -> lower cell
    ([0, 1, 9, 9.5, 10, 11], [0, 0, 1, 1, 2, 2], [0.5, 9.25, 10.5]),    # case C
    ([5, 1, 5, 3, 10, 11], [0, 0, 0, 0, 2, 2], [3.5, 5, 10.5]),         # case D: empty cell keeps its centroid
])
def test_hand_worked_cases(x, assign, mu):
    """tests/golden/cluster_hand.txt, cases A-D."""
    a, m = _hand(x)
    assert list(a) == assign
    assert np.allclose(m[:, 0], mu)


def test_hand_case_a_is_a_fixed_point_and_permutation():
    a, m = _hand([0, 4, 5, 6, 10, 11], n_iter=2)
    assert list(a) == [0, 1, 1, 1, 2, 2] and np.allclose(m[:, 0], [0, 5, 10.5])
    perm, sizes = orc.cluster_permutation(a, 3, 8)
    assert list(perm) == [0, 1, 2, 3, 4, 5, 6, 7] and list(sizes) == [1, 3, 2]


def test_cell_centres_on_a_ragged_lattice():
    """tests/golden/cluster_hand.txt: centre tokens of a 3 x 4 x 5 lattice cut into 2 x 2 x 2 cells."""
    grid, cell = (3, 4, 5), (2, 2, 2)
    x = np.arange(60, dtype=np.float64)[:, None]  # embedding = flat token index
    mu = orc.initial_centroids(x, grid, cell)
    CT, CH, CW = orc.cell_counts(grid, cell)
    assert (CT, CH, CW) == (2, 2, 3)
    flat = lambda t, h, w: (t * CH + h) * CW + w
    assert mu[flat(0, 0, 0), 0] == 0 and mu[flat(1, 1, 2), 0] == 54
    assert mu[flat(0, 1, 1), 0] == 12 and mu[flat(1, 0, 2), 0] == 44


def test_whole_grid_window_is_one_lloyd_step():
    """A window that covers every cell turns Eq. (5) into the plain nearest-
    centroid assignment: compare with scipy's vector quantiser, and the
    update with the mean of each code's members."""
    rng = np.random.default_rng(5)
    grid, cell = (3, 4, 6), (1, 2, 3)
    x = rng.standard_normal((72, 8))
    mu0 = orc.initial_centroids(x, grid, cell)
    a, mu = orc.local_window_clustering(x, grid, cell, (7, 5, 5), 1)
    code, _ = vq(x, mu0)
    assert np.array_equal(a, code)
    for u in range(mu0.shape[0]):
        members = x[code == u]
        expect = members.mean(axis=0) if len(members) else mu0[u]
        assert np.allclose(mu[u], expect)


def test_local_window_restricts_candidates():
    """Each token's centroid lies inside the window of its own cell."""
    rng = np.random.default_rng(6)
    grid, cell, window = (4, 6, 8), (2, 2, 2), (1, 3, 3)
    x = rng.standard_normal((192, 4))
    a, _ = orc.local_window_clustering(x, grid, cell, window, 3)
    g = orc.token_cells(grid, cell)
    counts = orc.cell_counts(grid, cell)
    CT, CH, CW = counts
    for l in range(192):
        u = g[l]
        assert a[l] in orc.window_cells((u // (CH * CW), (u // CW) % CH, u % CW), counts, window)


def test_objective_never_increases():
    """Every token's window contains its current centroid and a mean minimises
    a cluster's squared error, so the objective cannot grow between
    iterations."""
    rng = np.random.default_rng(7)
    grid, cell, window = (4, 6, 8), (2, 2, 4), (3, 3, 3)
    x = rng.standard_normal((192, 6))
    prev = np.inf
    for it in range(1, 6):
        a, mu = orc.local_window_clustering(x, grid, cell, window, it)
        obj = orc.clustering_objective(x, a, mu)
        assert obj <= prev + 1e-9
        prev = obj


def test_permutation_is_stable_and_inverse():
    rng = np.random.default_rng(8)
    a = rng.integers(0, 5, size=40)
    perm, sizes = orc.cluster_permutation(a, 6, 48)
    assert sorted(perm.tolist()) == list(range(48))
    assert list(sizes) == [int((a == u).sum()) for u in range(6)]
    pa = a[perm[:40]]
    assert np.all(np.diff(pa) >= 0)
    for u in range(5):
        toks = perm[:40][pa == u]
        assert np.all(np.diff(toks) > 0)   # original order kept inside a cluster
    y = rng.standard_normal((48, 3))
    assert np.array_equal(orc.unpermute_rows(orc.permute_rows(y, perm), perm), y)


def test_single_token_cells_leave_the_path_unchanged():
    """Cells of one token and a one-cell window: every token is its own
    cluster, the permutation is the identity and the clustered path is the
    plain path."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    res = orc.forward_clustered(q, k, v, w, (1, 1, 1), (1, 1, 1), 2)
    base = orc.forward(q, k, v, w)
    n = w.n_pad
    assert np.array_equal(res["perm_q"][0, 0], np.arange(n)) and np.array_equal(res["perm_k"][0, 1], np.arange(n))
    assert np.allclose(res["O"], base["O"]) and np.allclose(res["LSE"], base["LSE"], equal_nan=True)


def test_dense_selection_is_invariant_to_the_permutation():
    """With every key block kept, attention is a softmax over all keys, which
    no reordering of the keys changes, and the output is put back in token
    order: the clustered path equals brute-force dense attention."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)

    d = dataclasses.replace(w, cum_mass=0.0, fixed_k=w.n_pad // w.bk, n_anchor=0, micro_mode=0)
    res = orc.forward_clustered(q, k, v, d, (2, 2, 2), (3, 3, 3), 2)
    assert not np.array_equal(res["perm_q"][0, 0], np.arange(w.n_pad))  # the clustering did reorder
    mask = np.ones((w.n_pad, w.n_pad), dtype=bool)
    mask[:, w.n_valid:] = False
    mask[w.n_valid:, :] = False
    O, L = orc.masked_attention_bruteforce(q, k, v, np.broadcast_to(mask, (w.B, w.H, w.n_pad, w.n_pad)), w.scale)
    assert np.allclose(res["O"], O, atol=1e-12)
    fin = np.isfinite(L)
    assert np.allclose(res["LSE"][fin], L[fin], atol=1e-12)


def test_hand_worked_merging():
    """tests/golden/cluster_hand.txt, "Hardware-aware merging"."""
    sq, sk = [3, 1, 2, 2], [2, 2, 4]
    kept = [np.array([0]), np.array([0]), np.array([1, 2]), np.array([2])]
    assert orc.total_cost([[0], [1], [2], [3]], sq, sk, kept, 4, 4) == 80
    g1 = orc.merge_clusters(sq, sk, kept, 4, 4, [[0, 1, 0, 1]])
    assert g1 == [[0, 1], [2], [3]] and orc.total_cost(g1, sq, sk, kept, 4, 4) == 64
    g2 = orc.merge_clusters(sq, sk, kept, 4, 4, [[0, 1, 0, 1], [1, 0, 0, 1]])
    assert g2 == [[0, 1], [2, 3]] and orc.total_cost(g2, sq, sk, kept, 4, 4) == 48


def test_merging_partitions_and_never_raises_the_cost():
    rng = np.random.default_rng(21)
    nq, nk = 60, 40
    sq = rng.integers(0, 200, size=nq)
    sk = rng.integers(1, 200, size=nk)
    kept = [np.sort(rng.choice(nk, size=int(rng.integers(1, 12)), replace=False)) for _ in range(nq)]
    sides = rng.integers(0, 2, size=(8, nq))
    prev = orc.total_cost([[i] for i in range(nq)], sq, sk, kept, 128, 128)
    for r in range(1, 9):
        groups = orc.merge_clusters(sq, sk, kept, 128, 128, sides[:r])
        assert sorted(i for g in groups for i in g) == list(range(nq))
        cost = orc.total_cost(groups, sq, sk, kept, 128, 128)
        assert cost <= prev
        prev = cost
    assert prev < orc.total_cost([[i] for i in range(nq)], sq, sk, kept, 128, 128)


def test_cluster_selection_with_equal_sizes_is_top_k_of_the_logits():
    """With every key cluster the same size, Eq. (2)'s weights are a common
    factor and fixed-k selection keeps the k largest centroid logits."""
    rng = np.random.default_rng(22)
    muq, muk = rng.standard_normal((5, 8)), rng.standard_normal((9, 8))
    kept = orc.select_clusters(muq, muk, [3, 0, 4, 4, 1], [7] * 9, 0.3, 0, 0.0, 4)
    for i in range(5):
        expect = [] if i == 1 else sorted(np.argsort(-(muq[i] @ muk.T), kind="stable")[:4].tolist())
        assert kept[i].tolist() == expect


def test_cluster_blocks_with_everything_kept_is_dense_attention():
    """Every key cluster kept (fixed k = all): each token attends to all keys,
    whatever the clusters and the merging, so the result is dense attention."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    G = int(np.prod(orc.cell_counts(w.grid, (2, 2, 2))))
    sides = np.random.default_rng(3).integers(0, 2, size=(w.B, w.H, 4, G))
    res = orc.forward_cluster_blocks(q, k, v, w.n_valid, w.grid, (2, 2, 2), (3, 3, 3), 2, w.scale, 0, 0.0, G,
                                     sides=sides)
    assert any(len(g) > 1 for g in res["heads"][0]["groups"])
    mask = np.ones((w.n_pad, w.n_pad), dtype=bool)
    O, L = orc.masked_attention_bruteforce(q, k, v, np.broadcast_to(mask, (w.B, w.H, w.n_pad, w.n_pad)), w.scale)
    assert np.allclose(res["O"], O, atol=1e-12) and np.allclose(res["LSE"], L, atol=1e-12)


@pytest.mark.parametrize("lattice,grid,n_cells", [
    ((33, 45, 80), (11, 5, 5), 432),     # HunyuanVideo, Q grid
    ((33, 45, 80), (11, 3, 3), 1215),    # HunyuanVideo, K grid
    ((21, 45, 80), (7, 6, 6), 336),      # Wan 2.2, Q grid
    ((21, 45, 80), (6, 4, 4), 960),      # Wan 2.2, K grid
])
def test_cell_counts_match_the_published_centroid_counts(lattice, grid, n_cells):
    """HyperVAttention App. A.1, Table 2 lists the grid sizes and the
    resulting centroid counts N_q / N_k of each model's token lattice (81
    frames at 720p: 21 x 45 x 80 latent tokens; 129 frames: 33 x 45 x 80);
    the ceil cell count of reading C1 must reproduce every one of them, and
    the initial centroids are one per cell."""
    counts = orc.cell_counts(lattice, grid)
    assert int(np.prod(counts)) == n_cells
    assert int(np.prod(lattice)) in (75_600, 118_800)
    cells = orc.token_cells(lattice, grid)
    assert cells.min() == 0 and cells.max() == n_cells - 1
    assert np.unique(cells).size == n_cells                 # every cell holds a token


def test_local_window_search_space_reduction_is_six_point_three():
    """HyperVAttention §4.1: for HunyuanVideo (n = 118.8K tokens, N_c = 1215
    key centroids) a (3, 8, 8) window cuts the per-token search space 6.3x.
    With reading C3 an interior cell's window holds 3 * 8 * 8 = 192 cells,
    and 1215 / 192 rounds to 6.3; a cell at the lattice corner sees fewer."""
    lattice, grid, window = (33, 45, 80), (11, 3, 3), (3, 8, 8)
    counts = orc.cell_counts(lattice, grid)
    n_c = int(np.prod(counts))
    assert n_c == 1215
    interior = orc.window_cells((1, 7, 13), counts, window)
    assert interior.size == 192
    assert round(n_c / interior.size, 1) == 6.3
    corner = orc.window_cells((0, 0, 0), counts, window)
    assert corner.size == 2 * 5 * 5       # offsets 0..1 in t, 0..4 in h and w once clipped
