"""fp64 CPU oracle of 3D local-window clustering and the cluster permutation.

TEST INFRASTRUCTURE.  Like vsa_oracle, this file is the independent statement
of what the CUDA library computes, used only by the tests, the package smoke
check and the benchmark's CPU-baseline leg.  It shares no code with the CUDA
path.  Plain NumPy in float64.

Source: HyperVAttention: Efficient Sparse Attention with Spatio-Temporal
Clustering for Video Diffusion (arXiv 2607.03012v1), "HVA" below:

* §2 Eq. (1): the query and key tokens are reordered by permutations Pi^q
  and Pi^k so that the tokens of a cluster are contiguous (V follows K);
* §2 Eq. (4): attention runs on the reordered tensors and the output is put
  back in token order, O = (Pi^q)^-1 O';
* §4.1 Eq. (5): the T x H x W token lattice is cut into regular cells of
  (k_t, k_h, k_w) tokens, one centroid per cell, initialised from the token
  at the centre of the cell; a token is assigned to the nearest (squared
  Euclidean) centroid among the cells of a (w_t, w_h, w_w) window around its
  own cell; a centroid is then the mean of the tokens assigned to it; the
  cells never move, and the two steps repeat.

Readings taken where the page is silent (listed in the design notes too):

 C1 cell counts per axis are ceil(T / k_t) etc.; a cell at the far edge of
    an axis holds the remaining tokens;
 C2 the "token at the centre" of a cell with extent e along an axis is at
    offset (e - 1) // 2 from the cell's start (the lower middle);
 C3 the window of w cells along an axis spans cell offsets
    -((w - 1) // 2) .. w // 2 around the token's cell, clipped to the grid
    (symmetric for odd w; one more cell on the far side for even w);
 C4 ties in the assignment go to the lower flat cell index (t-major, then h,
    then w);
 C5 a centroid that receives no token keeps its previous value;
 C6 one iteration = assignment of every token, then the centroid update;
    the returned assignment is that of the last iteration and the returned
    centroids are those of its update;
 C7 within a cluster the permutation keeps the original token order, and the
    clusters follow each other in flat cell order; padding rows (at or past
    N_valid) stay where they are;
 C8 blocks of the permuted sequence are the attention blocks: the permuted
    Q', K', V' go through the same pooling, selection and attention as the
    unpermuted path (fixed block sizes).  Cluster-aligned variable blocks
    (padding or merging clusters to tile sizes, HVA §4.3) are a later step.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

__all__ = [
    "cell_counts", "token_cells", "initial_centroids", "window_offsets", "window_cells",
    "local_window_clustering", "clustering_objective", "cluster_permutation", "permute_rows",
    "unpermute_rows", "forward_clustered", "select_clusters", "tile_cost", "merge_clusters", "total_cost",
    "forward_cluster_blocks", "attend_cluster_groups", "lowe_ratio", "ambiguous_subset", "hybrid_anchor",
    "hybrid_update",
]


def cell_counts(grid: Sequence[int], cell: Sequence[int]) -> Tuple[int, int, int]:
    """Cells per axis (reading C1)."""
    return tuple(-(-g // c) for g, c in zip(grid, cell))


def token_cells(grid, cell) -> np.ndarray:
    """g(l) of Eq. (5) for every token l of the T x H x W lattice in frame-first
    order, as a flat cell index (t-major)."""
    T, H, W = grid
    CT, CH, CW = cell_counts(grid, cell)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    ct, ch, cw = t // cell[0], h // cell[1], w // cell[2]
    return ((ct * CH + ch) * CW + cw).reshape(-1)


def initial_centroids(x: np.ndarray, grid, cell) -> np.ndarray:
    """One centroid per cell: the embedding of the cell's centre token
    (reading C2).  x: [N, d] with N = T*H*W in frame-first order."""
    T, H, W = grid
    CT, CH, CW = cell_counts(grid, cell)
    mu = np.zeros((CT * CH * CW, x.shape[1]))
    for ct in range(CT):
        for ch in range(CH):
            for cw in range(CW):
                start = (ct * cell[0], ch * cell[1], cw * cell[2])
                ext = (min(cell[0], T - start[0]), min(cell[1], H - start[1]), min(cell[2], W - start[2]))
                t, h, w = (s + (e - 1) // 2 for s, e in zip(start, ext))
                mu[(ct * CH + ch) * CW + cw] = x[(t * H + h) * W + w]
    return mu


def window_offsets(w: int) -> range:
    """Cell offsets of a window of w cells along one axis (reading C3)."""
    return range(-((w - 1) // 2), w // 2 + 1)


def window_cells(cell_coord, counts, window) -> np.ndarray:
    """Flat indices of the cells of the window around one cell, ascending."""
    CT, CH, CW = counts
    out = []
    for dt in window_offsets(window[0]):
        for dh in window_offsets(window[1]):
            for dw in window_offsets(window[2]):
                t, h, w = cell_coord[0] + dt, cell_coord[1] + dh, cell_coord[2] + dw
                if 0 <= t < CT and 0 <= h < CH and 0 <= w < CW:
                    out.append((t * CH + h) * CW + w)
    return np.array(sorted(out), dtype=np.int64)


def local_window_clustering(x: np.ndarray, grid, cell, window, n_iter: int) -> Tuple[np.ndarray, np.ndarray]:
    """HVA §4.1 Eq. (5), n_iter rounds of (assignment, centroid update).

    x: [N, d] token embeddings (N = T*H*W, frame-first order).  Returns the
    assignment a [N] (flat cell index of each token's centroid) and the
    centroids mu [n_cells, d].
    """
    x = np.asarray(x, dtype=np.float64)
    counts = cell_counts(grid, cell)
    CT, CH, CW = counts
    g = token_cells(grid, cell)
    mu = initial_centroids(x, grid, cell)
    a = np.zeros(x.shape[0], dtype=np.int64)
    # the tokens of each cell share one window
    cell_tokens = [np.nonzero(g == u)[0] for u in range(CT * CH * CW)]
    windows = [window_cells((u // (CH * CW), (u // CW) % CH, u % CW), counts, window) for u in range(CT * CH * CW)]
    for _ in range(n_iter):
        for u, toks in enumerate(cell_tokens):
            if toks.size == 0:
                continue
            cand = windows[u]
            diff = x[toks][:, None, :] - mu[cand][None, :, :]
            dist = np.einsum("tcd,tcd->tc", diff, diff)
            a[toks] = cand[np.argmin(dist, axis=1)]  # argmin keeps the first minimum: lower cell (C4)
        for u in range(mu.shape[0]):
            members = a == u
            if members.any():
                mu[u] = x[members].mean(axis=0)
    return a, mu


def clustering_objective(x: np.ndarray, a: np.ndarray, mu: np.ndarray) -> float:
    """Sum over tokens of the squared distance to the assigned centroid."""
    diff = np.asarray(x, dtype=np.float64) - mu[a]
    return float(np.einsum("nd,nd->", diff, diff))


def cluster_permutation(a: np.ndarray, n_cells: int, n_pad: int) -> Tuple[np.ndarray, np.ndarray]:
    """Pi of Eq. (1) as a gather index: row i of the permuted sequence is
    token perm[i].  Tokens of cluster 0 first, then cluster 1, ...; original
    order within a cluster; padding rows N..n_pad-1 stay in place (C7).
    Returns (perm [n_pad], sizes [n_cells])."""
    N = a.shape[0]
    order = np.argsort(a, kind="stable")
    perm = np.concatenate([order, np.arange(N, n_pad)]).astype(np.int64)
    sizes = np.bincount(a, minlength=n_cells).astype(np.int64)
    return perm, sizes


def permute_rows(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x' = Pi x along the token axis (the last-but-one axis for 2-D rows)."""
    return x[perm]


def unpermute_rows(y: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x = Pi^-1 y: row perm[i] of the result is row i of y (Eq. (4))."""
    out = np.empty_like(y)
    out[perm] = y
    return out


def forward_clustered(q, k, v, w, cell, window, n_iter, head_enable=None) -> Dict[str, object]:
    """Cluster Q and K per (batch, head), permute (Eq. (1)), run the
    unpermuted path's oracle (vsa_oracle.forward) on Q', K', V', and put O and
    LSE back in token order (Eq. (4)).  Reading C8."""
    from .vsa_oracle import forward
    B, H, n_pad, d = q.shape
    N = w.n_valid
    grid = w.grid
    n_cells = int(np.prod(cell_counts(grid, cell)))
    qp, kp, vp = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    perms = {"q": np.zeros((B, H, n_pad), dtype=np.int64), "k": np.zeros((B, H, n_pad), dtype=np.int64)}
    assign = {"q": np.zeros((B, H, N), dtype=np.int64), "k": np.zeros((B, H, N), dtype=np.int64)}
    for b in range(B):
        for h in range(H):
            for name, x in (("q", q), ("k", k)):
                a, _ = local_window_clustering(x[b, h, :N], grid, cell, window, n_iter)
                perm, _ = cluster_permutation(a, n_cells, n_pad)
                perms[name][b, h] = perm
                assign[name][b, h] = a
            qp[b, h] = permute_rows(q[b, h], perms["q"][b, h])
            kp[b, h] = permute_rows(k[b, h], perms["k"][b, h])
            vp[b, h] = permute_rows(v[b, h], perms["k"][b, h])
    res = forward(qp, kp, vp, w, head_enable=head_enable)
    O = np.empty_like(res["O"])
    L = np.empty_like(res["LSE"])
    for b in range(B):
        for h in range(H):
            O[b, h] = unpermute_rows(res["O"][b, h], perms["q"][b, h])
            L[b, h] = unpermute_rows(res["LSE"][b, h], perms["q"][b, h])
    return {"perm_q": perms["q"], "perm_k": perms["k"], "assign_q": assign["q"], "assign_k": assign["k"],
            "permuted": res, "O": O, "LSE": L}


# ---------------------------------------------------------------------------
# Cluster-aligned blocks (HVA §2 Eq. (2)-(4) on clusters, §4.3 Eq. (7)-(10),
# Algorithm 1 "Parallel Agglomerative Merging")
#
# Further readings (C9-C14):
#  C9  cluster-level selection is the path's selection on centroids: logits
#      S_ij = <mu_i^q, mu_j^k> / sqrt(d), weights s_j^k = key-cluster sizes,
#      the same Top-p / Min-kc / fixed-k rule and ties (R3, R4); a query
#      cluster with no token keeps nothing; anchors are not used;
#  C10 the random bipartition of round r is given as one bit per query
#      cluster (an input array); a group takes the bit of its lowest member;
#  C11 pi(A) = argmin over B of dC(A, B), ties to the group with the lower
#      lowest member; among the A that chose the same B the smallest dC wins,
#      ties to the lower lowest member; only dC < 0 is applied (Alg. 1 l.14);
#  C12 a group's query tokens are its clusters' tokens, clusters in ascending
#      index, each in its permutation order, padded to a multiple of tau_q;
#      groups follow each other in ascending lowest member;
#  C13 a key cluster occupies ceil(s_j / seg) segments of seg keys, clusters in
#      ascending index; the last segment of a cluster holds s_j mod seg keys
#      (the rest is padding, never attended);
#  C14 every query token of group S attends to the keys of the union of the
#      key clusters selected by S's members (chi(S) of Eq. (8)).
# ---------------------------------------------------------------------------

def select_clusters(mu_q, mu_k, sizes_q, sizes_k, scale, k_min, cum_mass, fixed_k):
    """C9: kept key clusters per query cluster (ascending arrays)."""
    from .vsa_oracle import size_weighted_probs, select_row
    S = (np.asarray(mu_q, dtype=np.float64) @ np.asarray(mu_k, dtype=np.float64).T) * scale
    P, w = size_weighted_probs(S, np.asarray(sizes_k, dtype=np.float64))
    kept = []
    for i in range(S.shape[0]):
        if sizes_q[i] <= 0:
            kept.append(np.zeros(0, dtype=np.int64))
        else:
            kept.append(select_row(w[i], P[i], k_min, cum_mass, fixed_k)[0])
    return kept


def tile_cost(sq: int, wk: int, tau_q: int, tau_k: int) -> int:
    """Eq. (7) / (8): CTA-aligned query rows times CTA-aligned packed keys."""
    return (tau_q * (-(-sq // tau_q))) * (tau_k * (-(-wk // tau_k)))


def merge_clusters(sizes_q, sizes_k, kept, tau_q: int, tau_k: int, sides) -> List[List[int]]:
    """Algorithm 1 (Eq. (9), (10)) with the bipartitions ``sides`` [R, N_q]
    (readings C10, C11).  Returns the groups (ascending member lists),
    ordered by their lowest member."""
    nq = len(sizes_q)
    sk = np.asarray(sizes_k, dtype=np.int64)
    groups = {i: [i] for i in range(nq)}              # keyed by lowest member
    chi = {i: set(int(j) for j in kept[i]) for i in range(nq)}
    sq = {i: int(sizes_q[i]) for i in range(nq)}
    wk = lambda keys: int(sum(sk[j] for j in keys))
    cost = lambda g: tile_cost(sq[g], wk(chi[g]), tau_q, tau_k)
    for r in range(len(sides)):
        leaders = sorted(groups)
        A = [g for g in leaders if sides[r][g] == 0]
        B = [g for g in leaders if sides[r][g] != 0]
        if not A or not B:
            continue
        choice = {}
        for a in A:
            best = None
            for b in B:
                merged = tile_cost(sq[a] + sq[b], wk(chi[a] | chi[b]), tau_q, tau_k)
                d = merged - cost(a) - cost(b)
                if best is None or d < best[0]:
                    best = (d, b)
            choice[a] = best
        accepted = {}
        for a in A:
            d, b = choice[a]
            if d < 0 and (b not in accepted or d < accepted[b][0]):
                accepted[b] = (d, a)
        for b, (d, a) in accepted.items():
            lead = min(a, b)
            other = b if lead == a else a
            groups[lead] = sorted(groups[a] + groups[b])
            chi[lead] = chi[a] | chi[b]
            sq[lead] = sq[a] + sq[b]
            del groups[other], chi[other], sq[other]
    return [groups[g] for g in sorted(groups)]


def total_cost(groups, sizes_q, sizes_k, kept, tau_q, tau_k) -> int:
    sk = np.asarray(sizes_k, dtype=np.int64)
    tot = 0
    for g in groups:
        keys = set()
        for i in g:
            keys |= set(int(j) for j in kept[i])
        tot += tile_cost(int(sum(sizes_q[i] for i in g)), int(sum(sk[j] for j in keys)), tau_q, tau_k)
    return tot


def attend_cluster_groups(q, k, v, aq, ak, kept, groups, scale, O, L, only=None) -> None:
    """C14 for one (batch, head): every query token of group S attends to the
    key tokens of the clusters in chi(S) (Eq. (4) on the groups).  q, k, v
    [N_pad, d]; aq, ak the token clusters [N_valid]; writes the rows of O
    [N_pad, d] and L [N_pad] that belong to the groups (all, or the group
    indices in ``only``)."""
    from .vsa_oracle import attention_rows
    for gi, g in enumerate(groups):
        if only is not None and gi not in only:
            continue
        rows = np.nonzero(np.isin(aq, g))[0]
        if rows.size == 0:
            continue
        sel = sorted(set().union(*[set(int(j) for j in kept[i]) for i in g]))
        keys = np.nonzero(np.isin(ak, sel))[0]
        o, lse = attention_rows(q[rows], k[keys], v[keys], scale)
        O[rows] = o
        L[rows] = lse


def forward_cluster_blocks(q, k, v, n_valid, grid, cell, window, n_iter, scale, k_min, cum_mass, fixed_k,
                           tau_q=128, tau_k=128, sides=None) -> Dict[str, object]:
    """The cluster-aligned pipeline, per (batch, head): cluster Q and K
    (Eq. (5)), select key clusters per query cluster on centroids (C9),
    merge query clusters (Algorithm 1, when ``sides`` is given), and attend
    each query token to the keys of its group's selected clusters (C14).
    Returns O [B, H, N_pad, d], LSE [B, H, N_pad] in token order plus the
    per-head clusters, selections and groups."""
    from .vsa_oracle import NEG_INF
    B, H, n_pad, d = q.shape
    O = np.zeros((B, H, n_pad, d))
    L = np.full((B, H, n_pad), NEG_INF)
    info = []
    for b in range(B):
        for h in range(H):
            aq, muq = local_window_clustering(q[b, h, :n_valid], grid, cell, window, n_iter)
            ak, muk = local_window_clustering(k[b, h, :n_valid], grid, cell, window, n_iter)
            G = muq.shape[0]
            sq = np.bincount(aq, minlength=G)
            sk = np.bincount(ak, minlength=G)
            kept = select_clusters(muq, muk, sq, sk, scale, k_min, cum_mass, fixed_k)
            groups = merge_clusters(sq, sk, kept, tau_q, tau_k, sides[b][h]) if sides is not None else \
                [[i] for i in range(G)]
            attend_cluster_groups(q[b, h], k[b, h], v[b, h], aq, ak, kept, groups, scale, O[b, h], L[b, h])
            info.append({"assign_q": aq, "assign_k": ak, "mu_q": muq, "mu_k": muk, "sizes_q": sq, "sizes_k": sk,
                         "kept": kept, "groups": groups})
    return {"O": O, "LSE": L, "heads": info}


# ---------------------------------------------------------------------------
# Hybrid clustering across denoising steps (HVA §4.2, Eq. (6); App. A.1: full
# clustering every two steps, the 15% most ambiguous tokens cached)
#
# Further readings (C15-C19):
#  C15 Lowe's ratio rho_l = d1 / d2 (Eq. (6), Euclidean distances) is taken
#      over the centroids the token's last local assignment compared -- the
#      centroids of its window before the anchor step's final update -- with
#      u* that assignment's argmin (ties to the lower cell); a window of one
#      centroid gives rho = 0, d1 = d2 = 0 gives rho = 1;
#  C16 the cached subset is the ceil(frac * N) tokens of largest rho, ties to
#      the lower token index, listed in ascending token order;
#  C17 at an intermediate step each cached token is reassigned, with its
#      current embedding, to the nearest centroid of the whole current set
#      (squared Euclidean, ties to the lower cell); other tokens keep theirs;
#  C18 "updating the corresponding centroids": a cluster that gained or lost a
#      token is set to the mean of its members' current embeddings (an emptied
#      one keeps its centroid); every other centroid is unchanged;
#  C19 sizes and permutation follow the new assignment (C7).
# ---------------------------------------------------------------------------

def lowe_ratio(x: np.ndarray, mu: np.ndarray, grid, cell, window) -> np.ndarray:
    """C15: rho of every token against the centroids mu of its window."""
    x = np.asarray(x, dtype=np.float64)
    counts = cell_counts(grid, cell)
    CT, CH, CW = counts
    g = token_cells(grid, cell)
    rho = np.zeros(x.shape[0])
    for u in range(CT * CH * CW):
        toks = np.nonzero(g == u)[0]
        if toks.size == 0:
            continue
        cand = window_cells((u // (CH * CW), (u // CW) % CH, u % CW), counts, window)
        diff = x[toks][:, None, :] - mu[cand][None, :, :]
        dist = np.sqrt(np.einsum("tcd,tcd->tc", diff, diff))
        if cand.size == 1:
            continue  # rho = 0
        best = np.argmin(dist, axis=1)
        d1 = dist[np.arange(toks.size), best]
        rest = dist.copy()
        rest[np.arange(toks.size), best] = np.inf
        d2 = rest.min(axis=1)
        rho[toks] = np.where(d2 > 0, d1 / np.where(d2 > 0, d2, 1.0), 1.0)
    return rho


def ambiguous_subset(rho: np.ndarray, frac: float) -> np.ndarray:
    """C16: the ceil(frac * N) largest rho, ties to the lower index, ascending."""
    n = int(np.ceil(frac * rho.shape[0]))
    order = np.lexsort((np.arange(rho.shape[0]), -rho))
    return np.sort(order[:n])


def hybrid_anchor(x: np.ndarray, grid, cell, window, n_iter: int, frac: float):
    """An anchor step: full local-window clustering (n_iter >= 1 rounds), Lowe's
    ratio from the last round's comparison (C15) and the cached subset (C16).
    Returns (a, mu, rho, subset)."""
    a, mu = local_window_clustering(x, grid, cell, window, n_iter)
    _, mu_last = local_window_clustering(x, grid, cell, window, n_iter - 1) if n_iter > 1 else \
        (None, initial_centroids(np.asarray(x, dtype=np.float64), grid, cell))
    rho = lowe_ratio(x, mu_last, grid, cell, window)
    return a, mu, rho, ambiguous_subset(rho, frac)


def hybrid_update(x_new: np.ndarray, a_prev: np.ndarray, mu_prev: np.ndarray, subset: np.ndarray):
    """An intermediate step (C17, C18): returns (a, mu, changed clusters)."""
    x_new = np.asarray(x_new, dtype=np.float64)
    a = np.array(a_prev, dtype=np.int64, copy=True)
    mu = np.array(mu_prev, dtype=np.float64, copy=True)
    if subset.size:
        diff = x_new[subset][:, None, :] - mu_prev[None, :, :]
        dist = np.einsum("tcd,tcd->tc", diff, diff)
        a[subset] = np.argmin(dist, axis=1)  # first minimum: lower cell
    moved = subset[a[subset] != a_prev[subset]]
    changed = np.unique(np.concatenate([a_prev[moved], a[moved]])).astype(np.int64)
    for u in changed:
        members = a == u
        if members.any():
            mu[u] = x_new[members].mean(axis=0)
    return a, mu, changed
