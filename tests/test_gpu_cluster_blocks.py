"""GPU parity of the cluster-aligned blocks (HyperVAttention §2 Eq. (2)-(4) on
clusters, §4.3 Eq. (7)-(10), Algorithm 1) against the fp64 oracle, through
the C ABI.

Each stage is checked on the GPU's own inputs to that stage, so that a near
tie upstream (a token whose two best centroids are closer than fp32 rounding)
cannot make two correct results disagree downstream:
  * selection: the GPU's fp32 centroids and sizes go to the oracle's
    selection in fp64; rows decided by more than fp32 rounding must match
    bit-exactly, the rest must be valid selections (the same rule as the
    block selection tests);
  * merging: the GPU's kept lists and sizes go to the oracle's Algorithm 1;
    the groups must match exactly (integer arithmetic on both sides);
  * attention: the oracle attends every token to the keys of its group's
    clusters, with the GPU's assignment, groups and lists; O and LSE within
    the attention tolerances.
"""
import types

import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv

from gpu_helpers import assert_close_rows, compare_selection, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    yield
    assert vsa.read_device_status() == 0


def _clusters(x_dev, w, H, cell, window, iters):
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    params = vsa.ClusterParams.make(w.grid, cell, window, iters)
    G = vsa.cluster_count(params)
    a = torch.empty(w.B, H, w.n_valid, dtype=torch.int32, device="cuda")
    mu = torch.empty(w.B, H, G, w.d, device="cuda")
    sz = torch.empty(w.B, H, G, dtype=torch.int32, device="cuda")
    perm = torch.empty(w.B, H, w.n_pad, dtype=torch.int32, device="cuda")
    vsa.cluster_tokens(x_dev, shape, params, a, mu, sz, perm)
    return a, mu, sz, perm


def _oracle_select_with_info(mu_q, mu_k, sq, sk, scale, k_min, cum_mass, fixed_k):
    """Per-row kept lists and decision margins of the oracle's cluster selection."""
    S = (mu_q @ mu_k.T) * scale
    P, lw = orc.size_weighted_probs(S, sk.astype(np.float64))
    kept, info = [], []
    for i in range(S.shape[0]):
        if sq[i] <= 0:
            kept.append(np.zeros(0, dtype=np.int64))
            info.append({"m": 0, "m_p": 0, "gap": np.inf, "mass_margin": np.inf})
        else:
            kk, ii = orc.select_row(lw[i], P[i], k_min, cum_mass, fixed_k)
            kept.append(kk)
            info.append(ii)
    ref = orc.select_clusters(mu_q, mu_k, sq, sk, scale, k_min, cum_mass, fixed_k)
    assert all(np.array_equal(a, b) for a, b in zip(kept, ref))
    return kept, info, lw, P


CASES = [
    # name, heads, cell, window, iters, (k_min, cum_mass, fixed_k)
    ("tiny", None, (2, 2, 2), (3, 3, 3), 2, (2, 0.9, 0)),
    ("tiny", None, (1, 4, 3), (1, 2, 4), 2, (0, 0.0, 5)),
    ("wan13b", (0, 1), (3, 5, 8), (3, 5, 5), 3, (1, 0.95, 0)),
    ("hunyuan", (0, 1), (3, 5, 8), (3, 5, 5), 2, (0, 0.0, 198)),
]


def _gpu_select(w, heads, cell, window, iters, rule):
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    aq, muq, sq, pq = _clusters(to_dev(q), w, H, cell, window, iters)
    ak, muk, sk, pk = _clusters(to_dev(k), w, H, cell, window, iters)
    G = muq.shape[2]
    k_min, cum_mass, fixed_k = rule
    params = vsa.SelectParams(k_min=k_min, fixed_k=fixed_k, n_anchor=0, anchor_rot=0, cum_mass=cum_mass)
    counts = torch.empty(w.B, H, G, dtype=torch.int32, device="cuda")
    idx = torch.empty(w.B, H, G, G, dtype=torch.int32, device="cuda")
    vsa.select_clusters(muq, muk, sq, sk, w.scale, params, counts, idx)
    assert vsa.read_device_status() == 0
    return dict(q=q, k=k, v=v, H=H, G=G, aq=aq, ak=ak, muq=muq, muk=muk, sq=sq, sk=sk, pq=pq, pk=pk,
                counts=counts, idx=idx, rule=rule)


@pytest.mark.parametrize("name,heads,cell,window,iters,rule", CASES)
def test_select_clusters_matches_the_oracle(name, heads, cell, window, iters, rule):
    w = WORKLOADS[name]
    r = _gpu_select(w, heads, cell, window, iters, rule)
    H, G = r["H"], r["G"]
    k_min, cum_mass, fixed_k = rule
    kept = [[None] * H]
    info = [[None] * H]
    logw = [[None] * H]
    probs = [[None] * H]
    muq, muk = r["muq"].cpu().double().numpy(), r["muk"].cpu().double().numpy()
    sq, sk = r["sq"].cpu().numpy(), r["sk"].cpu().numpy()
    for h in range(H):
        kept[0][h], info[0][h], logw[0][h], probs[0][h] = _oracle_select_with_info(
            muq[0, h], muk[0, h], sq[0, h], sk[0, h], w.scale, k_min, cum_mass, fixed_k)
    rules = types.SimpleNamespace(n_k=G, n_anchor=0, anchor_rot=0, fixed_k=fixed_k, cum_mass=cum_mass)
    n_exact, n_near, _ = compare_selection(r["counts"].cpu().numpy(), r["idx"].cpu().numpy(), kept, info, logw,
                                           probs, rules)
    print(f"\n{name}: query clusters bit-exact {n_exact}, near-tie rows validity-checked {n_near}")
    assert n_exact >= 0.8 * (n_exact + n_near)
    # an empty query cluster keeps nothing
    assert np.all(r["counts"].cpu().numpy()[sq == 0] == 0)


def _gpu_merge(sq, sk, counts, idx, sides, tau_q, tau_k):
    """sq, sk int32 cuda [B, H, n]; sides uint8 numpy [B, H, R, n_q] or None."""
    B, H, nq = sq.shape
    nk = sk.shape[2]
    ws = torch.empty(vsa.merge_clusters_workspace_bytes(B * H, nq), dtype=torch.uint8, device="cuda")
    group_of = torch.empty(B, H, nq, dtype=torch.int32, device="cuda")
    g_counts = torch.empty(B, H, nq, dtype=torch.int32, device="cuda")
    g_idx = torch.full((B, H, nq, nk), -7, dtype=torch.int32, device="cuda")
    sides_d = None if sides is None else torch.from_numpy(np.ascontiguousarray(sides)).cuda()
    vsa.merge_clusters(sq, sk, counts, idx, sides_d, tau_q, tau_k, ws, group_of, g_counts, g_idx)
    assert vsa.read_device_status() == 0
    return group_of.cpu().numpy(), g_counts.cpu().numpy(), g_idx.cpu().numpy()


def _check_merge(sq, sk, counts, idx, sides, tau_q, tau_k, group_of, g_counts, g_idx):
    """The GPU's groups equal the oracle's Algorithm 1 on the same lists and bits."""
    B, H, nq = sq.shape
    n_merged = 0
    for b in range(B):
        for h in range(H):
            kept = [idx[b, h, i, :counts[b, h, i]].astype(np.int64) for i in range(nq)]
            s = sides[b, h] if sides is not None else np.zeros((0, nq), dtype=np.uint8)
            groups = orc.merge_clusters(sq[b, h], sk[b, h], kept, tau_q, tau_k, s)
            want = np.empty(nq, dtype=np.int64)
            for g in groups:
                want[g] = min(g)
            assert np.array_equal(group_of[b, h], want), (b, h)
            for g in groups:
                lead = min(g)
                union = sorted(set().union(*[set(kept[i].tolist()) for i in g]))
                assert g_counts[b, h, lead] == len(union)
                assert np.array_equal(g_idx[b, h, lead, :len(union)], union)
                n_merged += len(g) > 1
            lead_rows = np.zeros(nq, dtype=bool)
            lead_rows[[min(g) for g in groups]] = True
            assert np.all(g_counts[b, h, ~lead_rows] == 0)
            if len(s):
                c0 = orc.total_cost([[i] for i in range(nq)], sq[b, h], sk[b, h], kept, tau_q, tau_k)
                c1 = orc.total_cost(groups, sq[b, h], sk[b, h], kept, tau_q, tau_k)
                assert c1 <= c0
    return n_merged


@pytest.mark.parametrize("name,heads,cell,window,iters,rule,rounds,taus", [
    ("tiny", None, (2, 2, 2), (3, 3, 3), 2, (2, 0.9, 0), 3, (16, 16)),
    ("tiny", None, (1, 4, 3), (1, 2, 4), 2, (0, 0.0, 5), 0, (128, 128)),
    ("wan13b", (0, 2), (3, 5, 8), (3, 5, 5), 3, (1, 0.95, 0), 3, (128, 128)),
    ("wan13b", (0, 1), (3, 5, 8), (3, 5, 5), 3, (1, 0.95, 0), 4, (128, 96)),
])
def test_merge_clusters_on_gpu_lists_matches_the_oracle(name, heads, cell, window, iters, rule, rounds, taus):
    w = WORKLOADS[name]
    r = _gpu_select(w, heads, cell, window, iters, rule)
    sides = vsa_inputs_sides(w, rounds, r["G"], heads) if rounds else None
    out = _gpu_merge(r["sq"], r["sk"], r["counts"], r["idx"], sides, *taus)
    n = _check_merge(r["sq"].cpu().numpy(), r["sk"].cpu().numpy(), r["counts"].cpu().numpy(), r["idx"].cpu().numpy(),
                     sides, *taus, *out)
    print(f"\n{name}: merged groups {n}")
    if rounds and name == "wan13b":
        assert n > 0


def vsa_inputs_sides(w, rounds, G, heads):
    from video_inputs import merge_sides
    return merge_sides(w, rounds, G, heads)


@pytest.mark.parametrize("nq,nk,max_size,k_per_row,rounds,taus,seed", [
    (300, 257, 5000, 12, 4, (128, 128), 0),       # key sizes >= 2048: two digit passes
    (1024, 1024, 1 << 23, 6, 2, (64, 96), 1),     # maximum cluster counts, three digit passes
    (129, 64, 150, 40, 5, (32, 32), 2),           # one past a 128-group tile
])
def test_merge_clusters_synthetic_lists(nq, nk, max_size, k_per_row, rounds, taus, seed):
    """Merging on random sizes (zeros included) and random kept lists: tile
    boundaries of the pair contraction and every digit pass of the key sizes."""
    rng = np.random.default_rng(seed)
    B, H = 1, 2
    sq = rng.integers(0, 400, size=(B, H, nq)).astype(np.int32)
    sq[rng.random((B, H, nq)) < 0.05] = 0
    sk = rng.integers(0, max_size, size=(B, H, nk)).astype(np.int32)
    sk[rng.random((B, H, nk)) < 0.05] = 0
    counts = np.zeros((B, H, nq), dtype=np.int32)
    idx = np.full((B, H, nq, nk), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                if sq[b, h, i] == 0:
                    continue
                # rows near each other share most of their keys, as neighbouring clusters do
                base = (i * nk) // nq
                cand = np.unique(np.clip(base + rng.integers(-k_per_row, k_per_row + 1, size=k_per_row), 0, nk - 1))
                counts[b, h, i] = cand.size
                idx[b, h, i, :cand.size] = cand
    sides = rng.integers(0, 2, size=(B, H, rounds, nq)).astype(np.uint8)
    dev = lambda x: torch.from_numpy(x).cuda()
    out = _gpu_merge(dev(sq), dev(sk), dev(counts), dev(idx), sides, *taus)
    n = _check_merge(sq, sk, counts, idx, sides, *taus, *out)
    print(f"\nsynthetic nq={nq}: merged groups {n}")
    assert n > 0


def test_merge_clusters_rejects_bad_lists():
    B, H, nq, nk = 1, 1, 8, 8
    sq = torch.full((B, H, nq), 10, dtype=torch.int32, device="cuda")
    sk = torch.full((B, H, nk), 10, dtype=torch.int32, device="cuda")
    counts = torch.full((B, H, nq), 2, dtype=torch.int32, device="cuda")
    idx = torch.zeros(B, H, nq, nk, dtype=torch.int32, device="cuda")
    idx[..., 1] = 1
    idx[0, 0, 3, 1] = 0   # not strictly ascending
    ws = torch.empty(vsa.merge_clusters_workspace_bytes(B * H, nq), dtype=torch.uint8, device="cuda")
    outs = [torch.empty(B, H, nq, dtype=torch.int32, device="cuda") for _ in range(2)]
    g_idx = torch.empty(B, H, nq, nk, dtype=torch.int32, device="cuda")
    vsa.merge_clusters(sq, sk, counts, idx, None, 16, 16, ws, outs[0], outs[1], g_idx)
    assert vsa.read_device_status() == 5
    assert outs[1][0, 0, 3].item() == 0


def _run_cluster_blocks(w, heads, cell, window, iters, rule, rounds, taus=(128, 128)):
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    k_min, cum_mass, fixed_k = rule
    cfg = vsa.ClusterBlockConfig(n_valid=w.n_valid, lattice=w.grid, cell=cell, window=window, iters=iters,
                                 scale=w.scale, k_min=k_min, cum_mass=cum_mass, fixed_k=fixed_k, rounds=rounds,
                                 tau_q=taus[0], tau_k=taus[1])
    G = vsa.cluster_count(cfg.cluster_params())
    from video_inputs import merge_sides
    sides = torch.from_numpy(merge_sides(w, rounds, G, heads)).cuda() if rounds else None
    run = vsa.ClusterBlockAttention(cfg)
    b = run(to_dev(q), to_dev(k), to_dev(v), sides=sides)
    torch.cuda.synchronize()
    assert vsa.read_device_status() == 0
    host = {n: t.cpu() for n, t in b.items() if n not in ("q_rows", "kp", "vp", "o_rows", "merge_ws")}
    return q, k, v, H, G, host, (None if sides is None else sides.cpu().numpy())


def _groups_of(group_of_row):
    groups = {}
    for i, l in enumerate(group_of_row.tolist()):
        groups.setdefault(l, []).append(i)
    return [groups[l] for l in sorted(groups)]


def _check_plan(h, w, G, host, groups):
    """The query layout: every valid token on exactly one row, groups in
    leader order, members ascending, each cluster in permutation order, 128-row
    padding, tiles naming their group."""
    qmap, qinv = host["qmap"][0, h].numpy(), host["qinv"][0, h].numpy()
    tiles = host["tile_list"][0, h].numpy()
    sq = host["sizes_q"][0, h].numpy()
    perm = host["perm_q"][0, h].numpy()
    off = np.concatenate([[0], np.cumsum(sq)])
    row = 0
    for g in groups:
        n = int(sq[g].sum())
        want = np.concatenate([perm[off[i]:off[i + 1]] for i in g]) if n else np.zeros(0, dtype=np.int64)
        assert np.array_equal(qmap[row:row + n], want)
        pad = -(-n // 128) * 128
        assert np.all(qmap[row + n:row + pad] == -1)
        assert np.all(tiles[row // 128:(row + pad) // 128] == min(g))
        row += pad
    assert np.all(qmap[row:] == -2) and np.all(tiles[row // 128:] == -1)
    valid = qmap[qmap >= 0]
    assert np.array_equal(np.sort(valid), np.arange(w.n_valid))
    assert np.array_equal(qinv[valid], np.nonzero(qmap >= 0)[0])
    assert np.all(qinv[w.n_valid:] == -1)
    kc = host["kc_off"][0, h].numpy()
    assert np.array_equal(kc, np.concatenate([[0], np.cumsum(host["sizes_k"][0, h].numpy())[:-1]]))


@pytest.mark.parametrize("name,heads,cell,window,iters,rule,rounds,n_check", [
    ("tiny", None, (2, 2, 2), (3, 3, 3), 2, (2, 0.9, 0), 3, None),
    ("tiny", None, (1, 4, 3), (1, 2, 4), 2, (0, 0.0, 5), 0, None),      # no merging
    ("tiny", None, (1, 1, 1), (1, 3, 3), 1, (1, 0.5, 0), 3, None),      # one-token clusters
    ("wan13b", (3, 4), (3, 5, 8), (3, 5, 5), 3, (1, 0.95, 0), 3, 40),
])
def test_cluster_block_path_matches_the_oracle(name, heads, cell, window, iters, rule, rounds, n_check):
    w = WORKLOADS[name]
    q, k, v, H, G, host, sides = _run_cluster_blocks(w, heads, cell, window, iters, rule, rounds)
    for h in range(H):
        group_of = host["group_of"][0, h].numpy()
        groups = _groups_of(group_of)
        counts, idx = host["counts"][0, h].numpy(), host["idx"][0, h].numpy()
        kept = [idx[i, :counts[i]].astype(np.int64) for i in range(G)]
        # the merge on these lists is the oracle's
        s = sides[0, h] if sides is not None else np.zeros((0, G), dtype=np.uint8)
        assert [sorted(g) for g in groups] == orc.merge_clusters(host["sizes_q"][0, h].numpy(),
                                                                 host["sizes_k"][0, h].numpy(), kept, 128, 128, s)
        _check_plan(h, w, G, host, groups)
        # attention: the oracle on the GPU's assignment, lists and groups
        aq, ak = host["assign_q"][0, h].numpy(), host["assign_k"][0, h].numpy()
        O = np.zeros((w.n_pad, w.d))
        L = np.full(w.n_pad, -np.inf)
        if n_check is None:
            only = None
        else:
            rng = np.random.default_rng(7 + h)
            only = set(rng.choice(len(groups), size=min(n_check, len(groups)), replace=False).tolist())
            only |= {0, len(groups) - 1}
        orc.attend_cluster_groups(q[0, h].astype(np.float64), k[0, h].astype(np.float64),
                                  v[0, h].astype(np.float64), aq, ak, kept, groups, w.scale, O, L, only=only)
        og = host["o"][0, h].float().numpy()
        lg = host["lse"][0, h].numpy()
        if only is None:
            rows = np.arange(w.n_pad)
        else:
            rows = np.nonzero(np.isin(aq, [i for gi in only for i in groups[gi]]))[0]
            rows = np.concatenate([rows, np.arange(w.n_valid, w.n_pad)])
        assert_close_rows(og[None, None, rows], lg[None, None, rows], O[None, None, rows], L[None, None, rows],
                          [(0, 0, 0, rows.size)], bf16_out=True)
