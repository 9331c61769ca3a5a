"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks one oracle function against a closed form, a library
routine (torch scaled_dot_product_attention / logsumexp, numpy quantile and
sort), brute force over all subsets on tiny inputs, or a hand-worked value
stored under tests/golden with its citation.  A plausible slip in the oracle
(a dropped size weight, a wrong sign, a transposed operand, an off-by-one in a
rank) fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc
from video_inputs import WORKLOADS, make_qkv, micro_heads, round_to_bf16, sweep_points

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SDPA = torch.nn.functional.scaled_dot_product_attention


def _rand_qkv(rng, B, H, n_pad, d, n_valid):
    out = []
    for _ in range(3):
        x = round_to_bf16(rng.standard_normal((B, H, n_pad, d)).astype(np.float32))
        x[:, :, n_valid:] = 0
        out.append(x)
    return out


def _sdpa_masked(q, k, v, mask, scale):
    """Library reference: torch SDPA with a boolean mask, fp64; rows with no
    allowed key are returned as NaN by torch and are replaced by O = 0."""
    tq, tk, tv = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    tm = torch.from_numpy(mask)
    o = SDPA(tq, tk, tv, attn_mask=tm, scale=scale).numpy()
    logits = torch.einsum("bhnd,bhmd->bhnm", tq, tk) * scale
    logits = logits.masked_fill(~tm, float("-inf"))
    lse = torch.logsumexp(logits, dim=-1).numpy()
    empty = ~mask.any(axis=-1)
    o = np.where(empty[..., None], 0.0, o)
    return o, lse


# ---------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------

def test_pool_means_match_slice_means_with_padding():
    rng = np.random.default_rng(11)
    B, H, n_pad, d, n_valid, blk = 1, 2, 96, 8, 83, 16
    q, _, _ = _rand_qkv(rng, B, H, n_pad, d, n_valid)
    q[:, :, n_valid:] = 7.0          # padding rows must be ignored
    qbar = orc.pool_block_means(q, blk, n_valid)
    for i in range(n_pad // blk):
        r0, r1 = i * blk, min(i * blk + blk, n_valid)
        want = q[:, :, r0:r1].astype(np.float64).mean(axis=2) if r1 > r0 else 0.0
        np.testing.assert_allclose(qbar[:, :, i], want, rtol=0, atol=1e-12)
    assert list(orc.valid_counts(n_pad, blk, n_valid)) == [16, 16, 16, 16, 16, 3]


def test_pooled_logit_is_mean_of_token_logits():
    """Bilinearity: qbar_i . kbar_j equals the mean of q_a . k_b over the block pair."""
    rng = np.random.default_rng(12)
    B, H, n_pad, d, n_valid = 1, 1, 64, 16, 59
    q, k, _ = _rand_qkv(rng, B, H, n_pad, d, n_valid)
    bq, bk = 16, 8
    S = orc.block_logits(orc.pool_block_means(q, bq, n_valid), orc.pool_block_means(k, bk, n_valid), 0.5)
    tok = (q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T) * 0.5
    for i in range(n_pad // bq):
        for j in range(n_pad // bk):
            rows = range(i * bq, min(i * bq + bq, n_valid))
            cols = range(j * bk, min(j * bk + bk, n_valid))
            want = np.mean([tok[a, b] for a in rows for b in cols]) if len(rows) and len(cols) else 0.0
            assert abs(S[0, 0, i, j] - want) < 1e-12


# ---------------------------------------------------------------------------
# Eq. (2) size-weighted softmax
# ---------------------------------------------------------------------------

def test_size_weighted_softmax_equals_token_softmax_summed_per_block():
    """P'_ij equals the token-level softmax of the pooled logits (every valid
    key token of block j carries logit S_ij) summed over block j."""
    rng = np.random.default_rng(13)
    n_k, bk, n_valid = 6, 4, 21
    s = orc.valid_counts(n_k * bk, bk, n_valid)
    S = rng.normal(size=(3, n_k))
    P, w = orc.size_weighted_probs(S, s)
    for i in range(3):
        tok = np.array([S[i, t // bk] for t in range(n_valid)])
        e = np.exp(tok - tok.max())
        sm = e / e.sum()
        want = np.array([sm[j * bk:min(j * bk + bk, n_valid)].sum() for j in range(n_k)])
        np.testing.assert_allclose(P[i], want, rtol=1e-13, atol=1e-15)
    assert np.allclose(P.sum(axis=1), 1.0)


# ---------------------------------------------------------------------------
# Eq. (3) Top-p, Min-kc floor, fixed k, anchors
# ---------------------------------------------------------------------------

def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split("|")
            rows.append((lhs.split(), rhs.split()))
    return rows


def test_select_hand_worked_golden():
    qbar = np.array([[[[1.0]]]])
    kbar = np.array([[[[math.log(4.0)], [math.log(2.0)], [0.0], [math.log(2.0)]]]])
    for lhs, rhs in _read_golden("select_eq2_eq3_hand.txt"):
        k_min, p, fixed_k, n_anchor, rot = int(lhs[0]), float(lhs[1]), int(lhs[2]), int(lhs[3]), int(lhs[4])
        kept = orc.select_blocks(qbar, kbar, n_valid=7, bq=8, bk=2, scale=1.0, k_min=k_min, cum_mass=p,
                                 fixed_k=fixed_k, n_anchor=n_anchor, anchor_rot=rot)
        assert list(kept[0][0][0]) == [int(x) for x in rhs], (lhs, rhs, kept[0][0][0])


def _brute_top_p(P, p, k_min):
    """Minimal-cardinality subset with mass >= p (then the heaviest of that size),
    floored at k_min blocks, found by enumerating all subsets."""
    n = len(P)
    for size in range(0, n + 1):
        best = None
        for sub in itertools.combinations(range(n), size):
            mass = sum(P[j] for j in sub)
            if mass >= p and (best is None or mass > best[0]):
                best = (mass, sub)
        if best is not None:
            m = max(size, k_min)
            if m == size:
                return set(best[1])
            # floor: the m heaviest blocks
            return set(np.argsort(-P, kind="stable")[:m].tolist())
    return set(range(n))


@pytest.mark.parametrize("seed", range(8))
def test_top_p_matches_subset_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n_k = 7
    S = rng.normal(scale=1.5, size=(1, 1, 1, n_k))
    s = np.full(n_k, 4)
    P, _ = orc.size_weighted_probs(S[0, 0], s)
    for p in (0.3, 0.5, 0.77, 0.9, 0.99):
        for k_min in (0, 1, 3):
            # feed logits through select_blocks with d = 1: qbar = 1, kbar = S
            kept = orc.select_blocks(np.ones((1, 1, 1, 1)), S[0, 0, 0][None, None, :, None],
                                     n_valid=4 * n_k, bq=4 * n_k, bk=4, scale=1.0, k_min=k_min, cum_mass=p)
            got = set(kept[0][0][0].tolist())
            assert got == _brute_top_p(P[0], p, k_min)
            assert P[0][list(got)].sum() >= p - 1e-15


def test_top_p_special_cases_and_fixed_k():
    rng = np.random.default_rng(7)
    n_k = 12
    S = rng.normal(size=n_k)
    args = dict(n_valid=4 * n_k, bq=4 * n_k, bk=4, scale=1.0)
    one, kb = np.ones((1, 1, 1, 1)), S[None, None, :, None]
    assert len(orc.select_blocks(one, kb, cum_mass=1.0, **args)[0][0][0]) == n_k
    assert len(orc.select_blocks(one, kb, cum_mass=1e-9, k_min=3, **args)[0][0][0]) == 3
    got = orc.select_blocks(one, kb, fixed_k=5, **args)[0][0][0]
    assert set(got.tolist()) == set(np.argsort(-S)[:5].tolist())
    got = orc.select_blocks(one, kb, fixed_k=5, n_anchor=2, anchor_rot=3, **args)[0][0][0]
    assert set(got.tolist()) == set(np.argsort(-S)[:5].tolist()) | {3, 9}


# ---------------------------------------------------------------------------
# Eq. (4) attention over kept blocks
# ---------------------------------------------------------------------------

def _random_lists(rng, B, H, n_q, n_k, frac):
    return [[[np.sort(rng.choice(n_k, size=max(1, int(frac * n_k)), replace=False)) for _ in range(n_q)]
             for _ in range(H)] for _ in range(B)]


def test_all_blocks_kept_equals_dense_sdpa():
    rng = np.random.default_rng(21)
    B, H, n_pad, d, n_valid = 1, 2, 128, 32, 117
    q, k, v = _rand_qkv(rng, B, H, n_pad, d, n_valid)
    bq, bk = 32, 16
    kept = [[[np.arange(n_pad // bk) for _ in range(n_pad // bq)] for _ in range(H)] for _ in range(B)]
    O, L = orc.block_sparse_attention(q, k, v, kept, bq, bk, n_valid, 0.2)
    mask = np.zeros((B, H, n_pad, n_pad), dtype=bool)
    mask[:, :, :n_valid, :n_valid] = True
    Ow, Lw = _sdpa_masked(q, k, v, mask, 0.2)
    np.testing.assert_allclose(O[:, :, :n_valid], Ow[:, :, :n_valid], rtol=0, atol=1e-12)
    np.testing.assert_allclose(L[:, :, :n_valid], Lw[:, :, :n_valid], rtol=0, atol=1e-12)
    assert np.all(O[:, :, n_valid:] == 0) and np.all(np.isneginf(L[:, :, n_valid:]))


def test_block_sparse_equals_sdpa_with_token_mask_and_bruteforce():
    rng = np.random.default_rng(22)
    B, H, n_pad, d, n_valid = 1, 2, 256, 16, 250
    q, k, v = _rand_qkv(rng, B, H, n_pad, d, n_valid)
    bq, bk = 64, 32
    kept = _random_lists(rng, B, H, n_pad // bq, n_pad // bk, 0.4)
    O, L = orc.block_sparse_attention(q, k, v, kept, bq, bk, n_valid, 0.25)
    mask = orc.token_mask(kept, None, n_pad, bq, bk, n_valid)
    Ow, Lw = _sdpa_masked(q, k, v, mask, 0.25)
    Ob, Lb = orc.masked_attention_bruteforce(q, k, v, mask, 0.25)
    np.testing.assert_allclose(O, Ow, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Ob, Ow, rtol=0, atol=1e-12)
    fin = np.isfinite(Lw)
    np.testing.assert_allclose(L[fin], Lw[fin], rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lb[fin], Lw[fin], rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(L), ~fin)


def test_attention_rows_sum_to_one_and_lse_bounds():
    rng = np.random.default_rng(23)
    q = rng.normal(size=(5, 8))
    k = rng.normal(size=(37, 8))
    o, lse = orc.attention_rows(q, k, np.ones((37, 8)), 0.3)
    np.testing.assert_allclose(o, 1.0, atol=1e-14)
    logits = q @ k.T * 0.3
    assert np.all(lse >= logits.max(axis=1) - 1e-14)
    assert np.all(lse <= logits.max(axis=1) + math.log(37) + 1e-14)


# ---------------------------------------------------------------------------
# LSE merge
# ---------------------------------------------------------------------------

def test_lse_merge_hand_worked_golden():
    val = {"ln3": math.log(3.0), "ln4": math.log(4.0), "-inf": -math.inf}
    for lhs, rhs in _read_golden("lse_merge_hand.txt"):
        oa, la, ob, lb = (val.get(x, None) if x in val else float(x) for x in lhs)
        o, l = orc.lse_merge(np.array([[oa]]), np.array([la]), np.array([[ob]]), np.array([lb]))
        eo, el = (val.get(x, None) if x in val else float(x) for x in rhs)
        assert abs(o[0, 0] - eo) < 1e-14
        assert (np.isneginf(l[0]) and el == -math.inf) or abs(l[0] - el) < 1e-14


def test_merge_of_disjoint_supports_equals_union():
    rng = np.random.default_rng(31)
    B, H, n_pad, d, n_valid = 1, 1, 128, 16, 128
    q, k, v = _rand_qkv(rng, B, H, n_pad, d, n_valid)
    perm = rng.permutation(n_pad)
    ma = np.zeros((B, H, n_pad, n_pad), dtype=bool)
    mb = np.zeros_like(ma)
    ma[..., perm[:40]] = True
    mb[..., perm[40:90]] = True
    mb[:, :, :10, :] = False             # rows 0..9 only see support A
    Oa, La = _sdpa_masked(q, k, v, ma, 0.25)
    Ob, Lb = _sdpa_masked(q, k, v, mb, 0.25)
    Ou, Lu = _sdpa_masked(q, k, v, ma | mb, 0.25)
    O, L = orc.lse_merge(Oa, La, Ob, Lb)
    np.testing.assert_allclose(O, Ou, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lu, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Micro selection and the whole path
# ---------------------------------------------------------------------------

def test_micro_candidates_lie_in_omitted_blocks():
    kept = [0, 3]
    cand = orc.micro_candidates(kept, n_k=5, bk=64, micro_keys=16, n_valid=300)
    per = 4
    assert all((t // per) not in kept for t in cand)
    assert set(cand.tolist()) == {t for t in range(20) if (t // per) not in kept and t * 16 < 300}


def test_micro_topk_matches_rank_counting_brute_force():
    rng = np.random.default_rng(41)
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    n_valid = w.n_valid
    qbar = orc.pool_block_means(q, w.bq, n_valid)
    kbar = orc.pool_block_means(k, w.bk, n_valid)
    kept = orc.select_blocks(qbar, kbar, n_valid, w.bq, w.bk, w.scale, w.k_min, w.cum_mass)
    q64 = orc.pool_block_means(q, 64, n_valid)
    k16 = orc.pool_block_means(k, 16, n_valid)
    tiles = orc.select_micro_topk(q64, k16, kept, w.bq, w.bk, n_valid, w.scale, 4)
    S = (q64.astype(np.float64) @ np.swapaxes(k16, -1, -2)) * w.scale
    for h in range(w.H):
        for r in range(q64.shape[2]):
            i = r * 64 // w.bq
            cand = [t for t in range(k16.shape[2]) if (t * 16 // w.bk) not in set(kept[0][h][i].tolist())]
            # t is kept iff fewer than 4 candidates beat it (higher score, or equal score and lower index)
            want = [t for t in cand
                    if sum(1 for u in cand if S[0, h, r, u] > S[0, h, r, t]
                           or (S[0, h, r, u] == S[0, h, r, t] and u < t)) < 4]
            assert list(tiles[0][h][r]) == sorted(want)
    del rng


def test_micro_percentile_matches_numpy_quantile():
    rng = np.random.default_rng(42)
    H, n_r, n_t, d = 2, 12, 64, 8
    q64 = rng.normal(size=(1, H, n_r, d))
    k16 = rng.normal(size=(1, H, n_t, d))
    bq, bk = 128, 128
    n_valid = n_t * 16
    kept = [[[np.array([rng.integers(0, n_t * 16 // bk)]) for _ in range(n_r * 64 // bq)] for _ in range(H)]]
    tiles, info = orc.select_micro_percentile(q64, k16, kept, bq, bk, n_valid, 0.5, 0.9, np.array([1, 0]),
                                              with_info=True)
    inf0 = info[0][0]
    vals = inf0["S"][inf0["cand"]]
    tau = np.quantile(vals, 0.9, method="inverted_cdf")
    assert inf0["tau"] == tau
    n_sel = sum(len(t) for t in tiles[0][0])
    assert n_sel == inf0["M"] - math.ceil(0.9 * inf0["M"])       # no ties in continuous scores
    assert all(len(t) == 0 for t in tiles[0][1])                  # head 1 disabled
    assert orc.percentile_rank(0.99, 100) == 99 and orc.percentile_rank(0.99, 1000) == 990


@pytest.mark.parametrize("bq,bk,n_valid", [(64, 128, 1000), (128, 64, 1008), (64, 64, 1011), (128, 128, 1017)])
def test_micro_percentile_candidates_match_key_by_key_brute_force(bq, bk, n_valid):
    """The percentile mode's candidate set (HyMoR-Attn abstract: Micro tiles
    inside omitted blocks; reading R7) against an enumeration that decides
    every (Micro row, 16-key tile) pair key by key: the row must hold a valid
    query, every key of the tile must sit in a key block that the row's Macro
    query block omitted, and the tile must hold a valid key.  Query and key
    blocks of different sizes, 64-key blocks and a ragged last tile make a
    wrong block size in the tile-to-block map, a kept/omitted inversion or an
    off-by-one at n_valid fail here.  The selection is then every candidate
    strictly above the nearest-rank threshold, and nothing else."""
    rng = np.random.default_rng(bq + 7 * bk + n_valid)
    H, d = 2, 8
    n_pad = 1024
    n_r, n_t = n_pad // 64, n_pad // 16
    n_q, n_k = n_pad // bq, n_pad // bk
    q64 = rng.normal(size=(1, H, n_r, d))
    k16 = rng.normal(size=(1, H, n_t, d))
    kept = [[[np.sort(rng.choice(n_k, size=int(rng.integers(0, n_k)), replace=False)) for _ in range(n_q)]
             for _ in range(H)]]
    kept[0][0][0] = np.zeros(0, dtype=np.int64)              # a row that omitted everything
    kept[0][1][n_q - 1] = np.arange(n_k)                      # a row that kept everything
    tiles, info = orc.select_micro_percentile(q64, k16, kept, bq, bk, n_valid, 0.5, 0.75, np.array([1, 1]),
                                              with_info=True)
    for h in range(H):
        want = np.zeros((n_r, n_t), dtype=bool)
        for r in range(n_r):
            if r * 64 >= n_valid:
                continue
            macro_row = set(kept[0][h][(r * 64) // bq].tolist())
            for t in range(n_t):
                keys = range(16 * t, 16 * t + 16)
                want[r, t] = all((key // bk) not in macro_row for key in keys) and any(key < n_valid for key in keys)
        cand = info[0][h]["cand"]
        assert np.array_equal(cand, want), h
        S = (q64[0, h] @ k16[0, h].T) * 0.5
        vals = np.sort(S[want])
        tau = vals[math.ceil(0.75 * vals.size) - 1]
        sel = np.zeros_like(want)
        for r, t in enumerate(tiles[0][h]):
            sel[r, t] = True
        assert np.array_equal(sel, want & (S > tau)), h
        assert sel.sum() == vals.size - math.ceil(0.75 * vals.size)
    # the top-k mode builds its rows from the same rule
    topk = orc.select_micro_topk(q64, k16, kept, bq, bk, n_valid, 0.5, n_t)
    for h in range(H):
        for r in range(n_r):
            assert np.array_equal(topk[0][h][r], np.nonzero(info[0][h]["cand"][r])[0]), (h, r)


def test_tiny_forward_equals_sdpa_over_union_mask():
    """Whole path on the tiny workload: the merged output equals plain masked
    attention over the union of the Macro blocks and the Micro tiles."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    res = orc.forward(q, k, v, w, head_enable=micro_heads(w))
    mask = orc.token_mask(res["kept"], res["tiles"], w.n_pad, w.bq, w.bk, w.n_valid)
    macro = orc.token_mask(res["kept"], None, w.n_pad, w.bq, w.bk, w.n_valid)
    micro_only = mask & ~macro
    assert micro_only.sum() == sum(len(t) for t in res["tiles"][0][0] + res["tiles"][0][1]) * 64 * 16
    Ow, Lw = _sdpa_masked(q, k, v, mask, w.scale)
    np.testing.assert_allclose(res["O"], Ow, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["LSE"], Lw, rtol=0, atol=1e-12)
    # every row keeps at least the k_min floor and reaches the cum-mass
    for h in range(w.H):
        for i, info in enumerate(res["select_info"][0][h]):
            assert info["m"] >= w.k_min
            assert len(res["kept"][0][h][i]) >= 2


def test_workload_table_sizes():
    assert WORKLOADS["hunyuan"].n_valid == 118_800 and WORKLOADS["hunyuan"].n_pad == 118_912
    assert WORKLOADS["wan14b"].n_valid == 75_600 and WORKLOADS["wan14b"].n_pad == 75_776
    assert WORKLOADS["wan13b"].n_valid == 32_760 and WORKLOADS["wan13b"].n_pad == 32_768
    assert WORKLOADS["wan14b"].fixed_k == 89 and WORKLOADS["hunyuan"].fixed_k == 186
    assert [w.fixed_k for _, w in sweep_points()[:5]] == [929, 465, 232, 139, 74]
    assert int(micro_heads(WORKLOADS["hunyuan"]).sum()) == 6
