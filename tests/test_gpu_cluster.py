"""GPU parity of the cluster-permuted layout (HyperVAttention §4.1 Eq. (5),
§2 Eq. (1), (4)) against the fp64 clustering oracle, through the C ABI.

The assignment is an argmin of fp32 distances: a token whose two best
centroids are closer than fp32 rounding may legitimately pick either.  So
every round is checked on its own: given the centroids the GPU held before the
round (the library is deterministic, so a call with k-1 rounds reproduces
them), each token's GPU choice must be a nearest centroid of its window up to
a small tolerance, the centroids after the round must be the fp64 means of
the GPU's clusters, and the sizes and the permutation must be exactly those
the oracle derives from the GPU's assignment.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv

from gpu_helpers import assert_close_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    yield
    assert vsa.read_device_status() == 0


def _gpu_cluster(x_dev, w, H, cell, window, iters):
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    params = vsa.ClusterParams.make(w.grid, cell, window, iters)
    G = vsa.cluster_count(params)
    assert G == int(np.prod(orc.cell_counts(w.grid, cell)))
    a = torch.empty(w.B, H, w.n_valid, dtype=torch.int32, device="cuda")
    mu = torch.empty(w.B, H, G, w.d, device="cuda")
    sz = torch.empty(w.B, H, G, dtype=torch.int32, device="cuda")
    perm = torch.empty(w.B, H, w.n_pad, dtype=torch.int32, device="cuda")
    vsa.cluster_tokens(x_dev, shape, params, a, mu, sz, perm)
    assert vsa.read_device_status() == 0
    return a.cpu().numpy(), mu.cpu().numpy().astype(np.float64), sz.cpu().numpy(), perm.cpu().numpy(), G


def _check_round(x, grid, cell, window, mu_before, a, mu_after, sizes, perm, n_pad):
    """One round of Eq. (5) in fp64 against the GPU's result."""
    counts = orc.cell_counts(grid, cell)
    CT, CH, CW = counts
    g = orc.token_cells(grid, cell)
    G = CT * CH * CW
    n_near = 0
    for u in range(G):
        toks = np.nonzero(g == u)[0]
        cand = orc.window_cells((u // (CH * CW), (u // CW) % CH, u % CW), counts, window)
        assert np.all(np.isin(a[toks], cand)), "a token left its window"
        diff = x[toks][:, None, :] - mu_before[cand][None, :, :]
        dist = np.einsum("tcd,tcd->tc", diff, diff)
        best = dist.min(axis=1)
        chosen = dist[np.arange(toks.size), np.searchsorted(cand, a[toks])]
        scale = np.einsum("td,td->t", x[toks], x[toks]) + np.einsum("cd,cd->c", mu_before[cand],
                                                                    mu_before[cand]).max()
        tol = 1e-5 * scale + 1e-6
        assert np.all(chosen <= best + tol), (u, float((chosen - best).max()))
        n_near += int(np.sum(cand[dist.argmin(axis=1)] != a[toks]))
    # centroids: fp64 mean of the GPU's clusters; an empty cluster keeps its centroid
    for u in range(G):
        m = a == u
        expect = x[m].mean(axis=0) if m.any() else mu_before[u]
        assert np.allclose(mu_after[u], expect, rtol=2e-5, atol=2e-5), u
    assert np.array_equal(sizes, np.bincount(a, minlength=G))
    p_expect, _ = orc.cluster_permutation(a, G, n_pad)
    assert np.array_equal(perm, p_expect)
    return n_near


@pytest.mark.parametrize("name,heads,cell,window,iters", [
    ("tiny", None, (2, 2, 2), (3, 3, 3), 3),
    ("tiny", None, (1, 4, 3), (1, 2, 4), 2),            # ragged edge cells, even windows
    ("wan13b", (0, 1), (3, 5, 8), (3, 5, 5), 3),
])
def test_cluster_rounds_match_the_oracle(name, heads, cell, window, iters):
    w = WORKLOADS[name]
    q, k, _ = make_qkv(w, heads=heads)
    H = q.shape[1]
    for x_np in (q, k):
        xd = to_dev(x_np)
        prev = None
        for it in range(1, iters + 1):
            a, mu, sz, perm, G = _gpu_cluster(xd, w, H, cell, window, it)
            for h in range(H):
                x = x_np[0, h, :w.n_valid].astype(np.float64)
                mu_before = orc.initial_centroids(x, w.grid, cell) if prev is None else prev[1][0, h]
                n_near = _check_round(x, w.grid, cell, window, mu_before, a[0, h], mu[0, h], sz[0, h], perm[0, h],
                                      w.n_pad)
                assert n_near <= max(2, w.n_valid // 1000), n_near
            prev = (a, mu)
        # a second call gives the same result (deterministic)
        a2, mu2, _, perm2, _ = _gpu_cluster(xd, w, H, cell, window, iters)
        assert np.array_equal(a2, prev[0]) and np.array_equal(mu2, prev[1]) and np.array_equal(perm2, perm)


def test_permute_rows_gather_and_scatter():
    rng = np.random.default_rng(12)
    B, H, n_pad, d = 1, 3, 384, 128
    x = torch.from_numpy(rng.standard_normal((B, H, n_pad, d)).astype(np.float32)).cuda().to(torch.bfloat16)
    l = torch.from_numpy(rng.standard_normal((B, H, n_pad)).astype(np.float32)).cuda()
    perm = torch.from_numpy(np.stack([rng.permutation(n_pad) for _ in range(B * H)]).reshape(B, H, n_pad)
                            .astype(np.int32)).cuda()
    idx = perm.long()
    y = torch.empty_like(x)
    vsa.permute_rows(x, perm, y)
    assert torch.equal(y, torch.gather(x, 2, idx[..., None].expand(-1, -1, -1, d)))
    z = torch.empty_like(x)
    vsa.permute_rows(y, perm, z, inverse=True)
    assert torch.equal(z, x)
    ly = torch.empty_like(l)
    vsa.permute_rows(l, perm, ly)
    assert torch.equal(ly, torch.gather(l, 2, idx))
    assert vsa.read_device_status() == 0
    bad = perm.clone()
    bad[0, 1, 7] = n_pad + 3
    vsa.permute_rows(l, bad, ly)
    assert vsa.read_device_status() == 5


def test_clustered_path_tiny_matches_oracle_on_the_same_permutation():
    """The whole path in the cluster-permuted layout: the kernels' output equals
    the oracle's path run on the GPU's permutation (every row), and the GPU's
    clusters match the oracle's fp64 clustering except at near ties."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    cell, window, iters = (2, 2, 2), (3, 3, 3), 2
    cfg = vsa.PathConfig.from_workload(w)
    cfg.micro_mode = 0
    cfg.cluster_lattice, cfg.cluster_cell, cfg.cluster_window, cfg.cluster_iters = w.grid, cell, window, iters
    run = vsa.SparseVideoAttention(cfg)
    out = run(to_dev(q), to_dev(k), to_dev(v))
    assert vsa.read_device_status() == 0
    pq, pk = out["perm_q"].cpu().numpy(), out["perm_k"].cpu().numpy()
    qp, kp, vp = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for h in range(w.H):
        qp[0, h], kp[0, h], vp[0, h] = q[0, h][pq[0, h]], k[0, h][pk[0, h]], v[0, h][pk[0, h]]
    import dataclasses
    res = orc.forward(qp, kp, vp, dataclasses.replace(w, micro_mode=0))
    O = np.empty_like(res["O"])
    L = np.empty_like(res["LSE"])
    for h in range(w.H):
        O[0, h] = orc.unpermute_rows(res["O"][0, h], pq[0, h])
        L[0, h] = orc.unpermute_rows(res["LSE"][0, h], pq[0, h])
    assert_close_rows(out["o"].float().cpu().numpy(), out["lse"].cpu().numpy(), O, L,
                      [(0, h, 0, w.n_pad) for h in range(w.H)], bf16_out=True)
    # the clusters themselves, against fp64 clustering of the same tokens
    agree = 0
    for h in range(w.H):
        a_ref, _ = orc.local_window_clustering(q[0, h, :w.n_valid], w.grid, cell, window, iters)
        agree += int(np.sum(out["assign_q"][0, h].cpu().numpy() == a_ref))
    assert agree >= 0.99 * w.H * w.n_valid
