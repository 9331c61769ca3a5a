"""GPU parity of the hybrid clustering across denoising steps (HyperVAttention
§4.2, Eq. (6); readings C15-C19 of the clustering oracle) through the C ABI.

Each piece is checked on the GPU's own inputs to it:
  * Lowe's ratio against the oracle's ratio with the centroids the last
    assignment round compared (the library is deterministic, so a call with
    one round fewer reproduces them), inside the envelope that an fp32 error
    of the squared distances allows;
  * the cached subset exactly, on the GPU's own ratios (the n_sub largest,
    ties to the lower token);
  * an intermediate step: each cached token's new cluster is a nearest
    centroid of the whole set up to fp32 rounding (decided tokens exactly the
    oracle's), the touched centroids are the fp64 means of the GPU's clusters
    with the new embeddings, every other centroid is bit-for-bit unchanged,
    and sizes and permutation are exactly those of the GPU's assignment.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv, round_to_bf16

from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    yield
    assert vsa.read_device_status() == 0


def _buffers(w, H, G, n_sub):
    dev = "cuda"
    return dict(a=torch.empty(w.B, H, w.n_valid, dtype=torch.int32, device=dev),
                mu=torch.empty(w.B, H, G, w.d, device=dev),
                sz=torch.empty(w.B, H, G, dtype=torch.int32, device=dev),
                perm=torch.empty(w.B, H, w.n_pad, dtype=torch.int32, device=dev),
                rho=torch.empty(w.B, H, w.n_valid, device=dev),
                sub=torch.empty(w.B, H, n_sub, dtype=torch.int32, device=dev))


def _anchor(xd, w, H, cell, window, iters, frac):
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    params = vsa.ClusterParams.make(w.grid, cell, window, iters)
    G = vsa.cluster_count(params)
    n_sub = vsa.subset_size(w.n_valid, frac)
    b = _buffers(w, H, G, n_sub)
    vsa.cluster_anchor(xd, shape, params, b["a"], b["mu"], b["sz"], b["perm"], b["rho"], b["sub"])
    assert vsa.read_device_status() == 0
    return shape, params, G, n_sub, b


def _mu_of_last_round(xd, w, H, cell, window, iters):
    """Centroids the last assignment round compared: the state after iters - 1 rounds."""
    if iters == 1:
        return None
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    params = vsa.ClusterParams.make(w.grid, cell, window, iters - 1)
    G = vsa.cluster_count(params)
    b = _buffers(w, H, G, 1)
    vsa.cluster_tokens(xd, shape, params, b["a"], b["mu"], b["sz"], b["perm"])
    return b["mu"].cpu().double().numpy()


CASES = [("tiny", None, (2, 2, 2), (3, 3, 3), 2, 0.15),
         ("tiny", None, (1, 4, 3), (1, 2, 4), 1, 0.3),
         ("wan13b", (0, 1), (3, 5, 8), (3, 5, 5), 3, 0.15)]


@pytest.mark.parametrize("name,heads,cell,window,iters,frac", CASES)
def test_anchor_ratio_and_subset(name, heads, cell, window, iters, frac):
    w = WORKLOADS[name]
    q, _, _ = make_qkv(w, heads=heads)
    H = q.shape[1]
    xd = to_dev(q)
    shape, params, G, n_sub, b = _anchor(xd, w, H, cell, window, iters, frac)
    # the anchor's clusters are those of the plain clustering call
    ref = _buffers(w, H, G, 1)
    vsa.cluster_tokens(xd, shape, params, ref["a"], ref["mu"], ref["sz"], ref["perm"])
    for n in ("a", "mu", "sz", "perm"):
        assert torch.equal(b[n], ref[n]), n
    mu_last = _mu_of_last_round(xd, w, H, cell, window, iters)
    rho = b["rho"].cpu().numpy().astype(np.float64)
    sub = b["sub"].cpu().numpy()
    counts = orc.cell_counts(w.grid, cell)
    g = orc.token_cells(w.grid, cell)
    for h in range(H):
        x = q[0, h, :w.n_valid].astype(np.float64)
        mu = orc.initial_centroids(x, w.grid, cell) if mu_last is None else mu_last[0, h]
        want = orc.lowe_ratio(x, mu, w.grid, cell, window)
        # envelope of rho for an absolute error delta of each squared distance
        lo = np.zeros(w.n_valid)
        hi = np.ones(w.n_valid)
        for u in range(G):
            toks = np.nonzero(g == u)[0]
            cand = orc.window_cells((u // (counts[1] * counts[2]), (u // counts[2]) % counts[1], u % counts[2]),
                                    counts, window)
            if toks.size == 0 or cand.size < 2:
                lo[toks], hi[toks] = 0.0, 0.0
                continue
            d2 = np.sort(np.einsum("tcd,tcd->tc", x[toks][:, None] - mu[cand][None], x[toks][:, None] - mu[cand][None]),
                         axis=1)
            delta = 1e-5 * (np.einsum("td,td->t", x[toks], x[toks]) + np.einsum("cd,cd->c", mu[cand], mu[cand]).max())
            lo[toks] = np.sqrt(np.maximum(0, d2[:, 0] - delta) / (d2[:, 1] + delta))
            hi[toks] = np.sqrt((d2[:, 0] + delta) / np.maximum(d2[:, 1] - delta, 1e-30))
        r = rho[0, h]
        assert np.all(r >= np.minimum(lo, want) - 1e-6) and np.all(r <= np.maximum(hi, want) + 1e-6)
        assert np.all((r >= 0) & (r <= 1))
        # the subset, exactly, on the GPU's own ratios
        assert np.array_equal(sub[0, h], orc.ambiguous_subset(r, frac)), h


def _refine_and_check(xd_new, x_new, w, H, shape, params, G, b, ws):
    a_prev = b["a"].cpu().numpy().copy()
    mu_prev_t = b["mu"].clone()
    mu_prev = mu_prev_t.cpu().double().numpy()
    vsa.cluster_refine(xd_new, shape, params, b["sub"], b["a"], b["mu"], b["sz"], b["perm"], ws)
    assert vsa.read_device_status() == 0
    a = b["a"].cpu().numpy()
    mu = b["mu"].cpu().double().numpy()
    sub = b["sub"].cpu().numpy()
    n_moved = 0
    for h in range(H):
        x = x_new[0, h, :w.n_valid].astype(np.float64)
        s = sub[0, h].astype(np.int64)
        outside = np.setdiff1d(np.arange(w.n_valid), s)
        assert np.array_equal(a[0, h, outside], a_prev[0, h, outside])
        # each cached token: a nearest centroid of the whole set up to fp32 rounding
        diff = x[s][:, None, :] - mu_prev[0, h][None]
        dist = np.einsum("tcd,tcd->tc", diff, diff)
        chosen = dist[np.arange(s.size), a[0, h, s]]
        tol = 1e-5 * (np.einsum("td,td->t", x[s], x[s]) + np.einsum("cd,cd->c", mu_prev[0, h], mu_prev[0, h]).max())
        assert np.all(chosen <= dist.min(axis=1) + tol)
        a_ref, _, _ = orc.hybrid_update(x, a_prev[0, h], mu_prev[0, h], s)
        assert np.mean(a_ref[s] == a[0, h, s]) >= 0.999
        moved = s[a[0, h, s] != a_prev[0, h, s]]
        n_moved += moved.size
        touched = set(a_prev[0, h, moved].tolist()) | set(a[0, h, moved].tolist())
        for u in range(G):
            members = a[0, h] == u
            if u in touched and members.any():
                assert np.allclose(mu[0, h, u], x[members].mean(axis=0), rtol=2e-5, atol=2e-5), (h, u)
            else:
                assert np.array_equal(b["mu"][0, h, u].cpu(), mu_prev_t[0, h, u].cpu()), (h, u)
        assert np.array_equal(b["sz"][0, h].cpu().numpy(), np.bincount(a[0, h], minlength=G))
        p_ref, _ = orc.cluster_permutation(a[0, h], G, w.n_pad)
        assert np.array_equal(b["perm"][0, h].cpu().numpy(), p_ref)
    return n_moved


@pytest.mark.parametrize("name,heads,cell,window,iters,frac", CASES)
def test_refine_steps_match_the_oracle(name, heads, cell, window, iters, frac):
    w = WORKLOADS[name]
    q, _, _ = make_qkv(w, heads=heads)
    H = q.shape[1]
    shape, params, G, n_sub, b = _anchor(to_dev(q), w, H, cell, window, iters, frac)
    ws = torch.empty(vsa.cluster_refine_workspace_bytes(shape, params), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(5)
    x = q
    total = 0
    for step in range(2):  # two intermediate steps in a row
        x = round_to_bf16((x + 0.3 * rng.standard_normal(x.shape).astype(np.float32)).astype(np.float32))
        total += _refine_and_check(to_dev(x), x, w, H, shape, params, G, b, ws)
    print(f"\n{name}: cached tokens moved over two steps: {total}")
    assert total > 0


def test_cluster_block_path_over_anchor_and_refine_steps():
    """The cluster-aligned path on a refine step: its groups and lists come
    from the refined clusters, and O equals the oracle's attention over them."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    cfg = vsa.ClusterBlockConfig(n_valid=w.n_valid, lattice=w.grid, cell=(2, 2, 2), window=(3, 3, 3), iters=2,
                                 scale=w.scale, k_min=2, cum_mass=0.9, rounds=0)
    run = vsa.ClusterBlockAttention(cfg)
    with pytest.raises(ValueError):
        run(to_dev(q), to_dev(k), to_dev(v), cluster_step="refine")
    run(to_dev(q), to_dev(k), to_dev(v), cluster_step="anchor")
    rng = np.random.default_rng(9)
    q2, k2, v2 = (round_to_bf16((x + 0.3 * rng.standard_normal(x.shape).astype(np.float32)).astype(np.float32))
                  for x in (q, k, v))
    out = run(to_dev(q2), to_dev(k2), to_dev(v2), cluster_step="refine")
    torch.cuda.synchronize()
    assert vsa.read_device_status() == 0
    G = vsa.cluster_count(cfg.cluster_params())
    for h in range(w.H):
        aq, ak = out["assign_q"][0, h].cpu().numpy(), out["assign_k"][0, h].cpu().numpy()
        counts, idx = out["counts"][0, h].cpu().numpy(), out["idx"][0, h].cpu().numpy()
        kept = [idx[i, :counts[i]].astype(np.int64) for i in range(G)]
        groups = [[i] for i in range(G)]
        O = np.zeros((w.n_pad, w.d))
        L = np.full(w.n_pad, -np.inf)
        orc.attend_cluster_groups(q2[0, h].astype(np.float64), k2[0, h].astype(np.float64),
                                  v2[0, h].astype(np.float64), aq, ak, kept, groups, w.scale, O, L)
        og, lg = out["o"][0, h].float().cpu().numpy(), out["lse"][0, h].cpu().numpy()
        fin = np.isfinite(L)
        assert np.array_equal(fin, np.isfinite(lg))
        assert np.abs(lg[fin] - L[fin]).max() <= 1e-3
        assert np.all(np.abs(og - O) <= 1e-2 + np.abs(O) * 2.0 ** -8)
