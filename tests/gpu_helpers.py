"""Shared plumbing of the GPU parity tests: device copies of the seeded inputs,
per-head oracle evaluation, and the comparison rules.

Comparison rules (the same in every test):
  * integer outputs (kept lists, Micro lists, counts) are compared bit-exactly
    on every row whose selection boundary is decided by more than the fp32
    rounding of the kernel: log-weight gap at the cut >= GAP and cumulative-mass
    margin >= MASS.  A row closer than that to a tie has several correct
    answers; it must be one of them: with m' the number of non-anchor blocks
    the kernel kept (m' = m in fixed mode; m' within one of m, and different
    from m only at a cumulative-mass near-tie, in Top-p mode) and cut' the
    m'-th largest log-weight of the row, every kept non-anchor block has
    log-weight >= cut' - GAP, every omitted block <= cut' + GAP, the anchors
    are kept and, in Top-p mode, the kept mass reaches p - MASS.  Such rows
    are counted and the counts printed.
  * O within max-abs O_TOL and LSE within max-abs LSE_TOL of the fp64 oracle
    (bf16 inputs, fp32 accumulation, P rounded to bf16 before P.V) when O is
    written in fp32.  When O is written in bf16 the bound also carries the
    final rounding to bf16, at most half a bf16 ulp: |O| * 2^-8.
"""
import math

import numpy as np
import torch

import oracle as orc

GAP = 1e-4       # log-weight units; fp32 logit error of the kernel is ~1e-6
MASS = 1e-5      # cumulative-mass units
O_TOL = 1e-2
LSE_TOL = 1e-3


def to_dev(x: np.ndarray) -> torch.Tensor:
    """float32 array of bf16-representable values -> contiguous cuda bf16 (exact)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(torch.bfloat16).contiguous()


def oracle_select_per_head(q, k, w, heads=None):
    """Oracle pooling + selection, one head at a time (bounded memory).

    Returns kept[b][h][i], info[b][h][i], w_logweights[b][h] ([n_q, n_k]),
    P[b][h], and the pooled means (qbar, kbar) as float64 arrays."""
    B, H = q.shape[0], q.shape[1]
    heads = range(H) if heads is None else heads
    kept = [[None] * H for _ in range(B)]
    info = [[None] * H for _ in range(B)]
    logw = [[None] * H for _ in range(B)]
    probs = [[None] * H for _ in range(B)]
    qbar = np.zeros((B, H, w.n_pad // w.bq, w.d))
    kbar = np.zeros((B, H, w.n_pad // w.bk, w.d))
    s = orc.valid_counts(w.n_pad, w.bk, w.n_valid)
    for b in range(B):
        for h in heads:
            qb = orc.pool_block_means(q[b:b + 1, h:h + 1], w.bq, w.n_valid)
            kb = orc.pool_block_means(k[b:b + 1, h:h + 1], w.bk, w.n_valid)
            qbar[b, h], kbar[b, h] = qb[0, 0], kb[0, 0]
            kk, ii = orc.select_blocks(qb, kb, w.n_valid, w.bq, w.bk, w.scale, w.k_min, w.cum_mass, w.fixed_k,
                                       w.n_anchor, w.anchor_rot, with_info=True)
            kept[b][h], info[b][h] = kk[0][0], ii[0][0]
            P, lw = orc.size_weighted_probs(orc.block_logits(qb[0, 0], kb[0, 0], w.scale), s)
            logw[b][h], probs[b][h] = lw, P
    return kept, info, logw, probs, qbar, kbar


def compare_selection(gpu_counts, gpu_idx, kept, info, logw, probs, w, heads=None, gpu_mask=None):
    """Bit-exact comparison on decided rows, validity on near-tie rows.

    Returns (n_exact_rows, n_near_tie_rows, n_rows_gap_below_1e-3)."""
    B, H, n_q = gpu_counts.shape
    heads = range(H) if heads is None else heads
    anchors = set(orc.anchor_columns(w.n_k, w.n_anchor, w.anchor_rot))
    n_exact = n_near = n_1e3 = 0
    for b in range(B):
        for h in heads:
            for i in range(n_q):
                want = kept[b][h][i]
                c = int(gpu_counts[b, h, i])
                got = gpu_idx[b, h, i, :c]
                inf = info[b][h][i]
                assert np.all(np.diff(got) > 0), (b, h, i, "not ascending")
                if gpu_mask is not None:
                    row = np.zeros(w.n_k, dtype=np.uint8)
                    row[got] = 1
                    assert np.array_equal(gpu_mask[b, h, i], row)
                if inf["gap"] < 1e-3:
                    n_1e3 += 1
                decided = inf["gap"] >= GAP and inf["mass_margin"] >= MASS
                if decided:
                    n_exact += 1
                    assert c == len(want) and np.array_equal(got, want), (b, h, i, got, want, inf)
                    continue
                n_near += 1
                lw = logw[b][h][i]
                gs = set(got.tolist())
                m = inf["m"]
                assert anchors <= gs or m == 0, (b, h, i, "anchor missing")
                free = gs - anchors                     # blocks the ranking chose
                if w.fixed_k > 0:
                    # exactly m blocks of the ranking; some of them may be anchors
                    assert len(free) <= m <= len(gs), (b, h, i, len(gs), m)
                    m_gpu = m
                else:
                    m_gpu = len(free) if not anchors else m
                    assert abs(m_gpu - m) <= 1, (b, h, i, m_gpu, m)
                    if m_gpu != m:
                        assert inf["mass_margin"] < MASS, (b, h, i, "count differs without a mass tie")
                if m_gpu >= 1:
                    cut = np.sort(lw)[::-1][m_gpu - 1]
                    for j in free:
                        assert lw[j] >= cut - GAP, (b, h, i, j, lw[j], cut)
                    omitted = np.setdiff1d(np.arange(w.n_k), got)
                    if omitted.size:
                        assert lw[omitted].max() <= cut + GAP, (b, h, i, lw[omitted].max(), cut)
                if w.fixed_k == 0 and w.cum_mass > 0:
                    mass = float(probs[b][h][i][sorted(gs)].sum())
                    assert mass >= w.cum_mass - MASS, (b, h, i, mass)
    return n_exact, n_near, n_1e3


def sample_blocks(w, n, seed=0, heads=None):
    """A few (b, h, query block) triples: first, last (ragged) and random ones."""
    rng = np.random.default_rng(seed)
    H = w.H if heads is None else heads
    n_q = w.n_pad // w.bq
    last_valid = (w.n_valid - 1) // w.bq
    out = {(0, 0, 0), (0, H - 1, last_valid)}
    while len(out) < n:
        out.add((0, int(rng.integers(0, H)), int(rng.integers(0, n_q))))
    return sorted(out)


def assert_close_rows(O_gpu, L_gpu, O_ref, L_ref, rows, tol_o=O_TOL, tol_l=LSE_TOL, bf16_out=False):
    """Compare O / LSE on the given row ranges [(b, h, r0, r1)].  Returns the
    worst |dO| beyond the output-rounding allowance and the worst |dLSE|."""
    worst_o = worst_l = 0.0
    for b, h, r0, r1 in rows:
        og = O_gpu[b, h, r0:r1].astype(np.float64)
        lg = L_gpu[b, h, r0:r1].astype(np.float64)
        orf = O_ref[b, h, r0:r1]
        lrf = L_ref[b, h, r0:r1]
        fin = np.isfinite(lrf)
        assert np.array_equal(np.isfinite(lg), fin), (b, h, r0, "LSE finiteness differs")
        if fin.any():
            worst_l = max(worst_l, float(np.abs(lg[fin] - lrf[fin]).max()))
        allow = np.abs(orf) * 2.0 ** -8 if bf16_out else 0.0
        worst_o = max(worst_o, float((np.abs(og - orf) - allow).max()))
        assert np.all(og[~fin] == 0)
    assert worst_o <= tol_o, worst_o
    assert worst_l <= tol_l, worst_l
    return worst_o, worst_l


def percentile_margin_ok(info_head, tiles_row_oracle, r, delta=GAP):
    """Tiles of Micro row r whose oracle score is at least delta away from tau."""
    S, cand, tau = info_head["S"], info_head["cand"], info_head["tau"]
    far = cand[r] & (np.abs(S[r] - tau) >= delta)
    return far


def finite_or(x, v):
    return x if math.isfinite(x) else v
