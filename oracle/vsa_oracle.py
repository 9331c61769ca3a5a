"""fp64 CPU oracle of pooled block-sparse attention with a Micro residual.

TEST INFRASTRUCTURE.  This file is the independent statement of what the CUDA
library computes.  Only the tests, the package smoke check and the benchmark's
CPU-baseline leg use it; it shares no code, header, table or helper with the
CUDA path, and the CUDA path never imports it.  Everything here is plain NumPy
in float64 (inputs are bfloat16 values, widened exactly), written for a reader
to check against the pages by eye, not for speed.

Sources (pages by title; section / equation on the page):

* HyperVAttention: Efficient Sparse Attention with Spatio-Temporal Clustering
  for Video Diffusion (arXiv 2607.03012v1), "HVA" below:
    - §2 Eq. (2): centroid logits S_ij = <mu_i^q, mu_j^k> / sqrt(d) and the
      size-weighted softmax P'_ij = s_j exp(S_ij) / sum_o s_o exp(S_io);
    - §2 Eq. (3): row-wise Top-p = the smallest set of key indices, taken in
      descending P', whose cumulative probability is at least p;
    - §2 Eq. (4): attention restricted to the selected key blocks;
    - §4.1: a centroid is the mean of its tokens;
    - App. A.1 "Min-kc": a minimum number of key blocks is always kept even
      when Top-p is reached earlier.
* HyMoR-Attn: Granularity-Matched Repair of Omitted Attention Support for
  Video Diffusion (abstract): a coarse Macro block-sparse backbone, a fine
  Micro residual over tiles inside omitted blocks chosen online, and exact
  LSE merging of the two outputs.
* Rectified SpaAttn: Revisiting Attention Sparsity for Efficient Video
  Generation (abstract): block importance from pooled query-key interactions.
* LVSA (abstract on the "FreqFormer" page): rotating global anchor columns.
* MOD-DiT (arXiv 2601.11641), "Block-wise Attention Computation": Q and K are
  partitioned into non-overlapping blocks of a fixed size (128).

Readings taken where the pages are silent (each one is listed in the design
notes of the repository):

 R1 pooling is the mean over the block's valid tokens (HVA §4.1 centroids);
    a block with no valid token has mean 0;
 R2 s_j in Eq. (2) is the number of valid keys in key block j; a key block with
    s_j = 0 has P' = 0;
 R3 the ranking key is the log-weight w_ij = S_ij + ln s_j (same order as P');
    ties go to the lower key-block index;
 R4 Top-p (inclusive "at least p") is combined with the Min-kc floor as a
    union of prefixes of the same order: keep max(k_min, m_p) blocks; in fixed
    mode keep exactly min(k, n_k) blocks and ignore p;
 R5 anchors: n_anchor columns (rot + t * floor(n_k / n_anchor)) mod n_k,
    t = 0..n_anchor-1, are added to every non-empty row;
 R6 a query block with no valid row keeps nothing;
 R7 Micro rows are 64 query rows and Micro tiles 16 keys; a tile is a
    candidate for a Micro row iff its whole key range lies in a key block that
    the row's Macro query block omitted and it holds at least one valid key;
 R8 the Micro score is the pooled logit qbar64 . kbar16 / sqrt(d);
 R9 Micro top-k keeps the k highest-scoring candidates per Micro row (ties to
    the lower tile index); the per-head percentile mode keeps, in each enabled
    head, the candidates whose score is strictly above tau, the
    ceil(q * M)-th smallest of the head's M candidate scores (nearest rank,
    ceil evaluated in IEEE double);
 R10 LSE is the natural-log sum of exp of the scaled logits; an empty row has
    O = 0 and LSE = -inf, and the merge passes the other side through;
 R11 query rows at or beyond N_valid are padding: O = 0, LSE = -inf; keys at or
    beyond N_valid never contribute.

How each function is pinned to something other than itself (the pages print
no worked example, so the stored goldens are hand-worked from the equations;
tests/test_oracle_pins.py):
  pool_block_means       means of explicit slices, padding excluded;
  block_logits           the mean of the block's token logits (bilinearity);
  size_weighted_probs    the token-level softmax of pooled logits summed per
                         block (what the size weight stands for);
  select_row / _blocks   a hand-worked Eq. (2)-(3) golden, brute force over
                         all subsets (n_k <= 8), p -> 1 / p -> 0 / fixed-k
                         special cases, the selected-mass >= p invariant;
  block_sparse_attention dense SDPA (torch, fp64) when every block is kept,
                         SDPA under the token mask, brute force, rows of P
                         summing to one and LSE above the row maximum;
  lse_merge              a hand-worked golden, disjoint supports merging to
                         attention over their union, an empty side passing
                         the other through;
  micro_candidates /     candidates inside omitted blocks only, and (for both
  select_micro_*         modes, which build their rows from micro_candidates)
                         a key-by-key enumeration of every (row, tile) pair
                         with query and key blocks of different sizes and a
                         ragged last tile; top-k against a rank-counting
                         brute force, the percentile against numpy's
                         quantile (nearest rank);
  forward                the tiny layer equal to SDPA over the union of the
                         Macro and Micro token masks.
No function here is parity-unpinned.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "valid_counts", "pool_block_means", "block_logits", "size_weighted_probs", "rank_order",
    "select_row", "select_blocks", "anchor_columns", "block_sparse_attention",
    "attention_rows", "micro_candidates", "micro_scores", "select_micro_topk",
    "select_micro_percentile", "percentile_rank", "micro_attention", "lse_merge", "token_mask",
    "masked_attention_bruteforce", "forward", "lists_to_mask",
]

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# a1: pooling (HVA §4.1 centroid = mean; Rectified SpaAttn pooled Q/K)
# ---------------------------------------------------------------------------

def valid_counts(n_pad: int, block: int, n_valid: int) -> np.ndarray:
    """Number of valid tokens in each block of ``block`` rows (reading R1/R2)."""
    nb = n_pad // block
    starts = np.arange(nb, dtype=np.int64) * block
    return np.clip(n_valid - starts, 0, block).astype(np.int64)


def pool_block_means(x: np.ndarray, block: int, n_valid: int) -> np.ndarray:
    """Block means of x [B, H, N_pad, d] over valid rows -> [B, H, nb, d] float64.

    HVA §4.1: a centroid is the average of the embeddings assigned to it; here
    the "cluster" of a block is its valid tokens in the original frame-first
    layout (MOD-DiT "Block-wise Attention Computation").
    """
    B, H, n_pad, d = x.shape
    nb = n_pad // block
    xv = np.array(x, dtype=np.float64, copy=True)
    xv[:, :, n_valid:, :] = 0.0
    sums = xv.reshape(B, H, nb, block, d).sum(axis=3)
    cnt = valid_counts(n_pad, block, n_valid)
    out = np.zeros_like(sums)
    nz = cnt > 0
    out[:, :, nz, :] = sums[:, :, nz, :] / cnt[nz][None, None, :, None]
    return out


# ---------------------------------------------------------------------------
# a2: pooled logits and size-weighted softmax (HVA §2 Eq. (2))
# ---------------------------------------------------------------------------

def block_logits(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """S_ij = <qbar_i, kbar_j> * scale for every (i, j): [..., n_q, n_k]."""
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) * scale


def size_weighted_probs(S: np.ndarray, s: np.ndarray):
    """Eq. (2): P'_ij = s_j exp(S_ij) / sum_o s_o exp(S_io).

    Returns (P', w) where w_ij = S_ij + ln s_j is the log-weight (-inf where
    s_j = 0), the ranking key of reading R3.
    """
    s = np.asarray(s, dtype=np.float64)
    with np.errstate(divide="ignore"):
        logs = np.where(s > 0, np.log(np.maximum(s, 1e-300)), NEG_INF)
    w = S + logs
    m = np.max(w, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(w - m)
    z = e.sum(axis=-1, keepdims=True)
    P = np.where(z > 0, e / np.where(z > 0, z, 1.0), 0.0)
    return P, w


def rank_order(w_row: np.ndarray) -> np.ndarray:
    """Key-block indices in descending log-weight, ties to the lower index (R3)."""
    n = w_row.shape[0]
    return np.lexsort((np.arange(n), -w_row))


# ---------------------------------------------------------------------------
# a3: selection (HVA §2 Eq. (3) Top-p, App. A.1 Min-kc, LVSA anchors)
# ---------------------------------------------------------------------------

def anchor_columns(n_k: int, n_anchor: int, rot: int) -> List[int]:
    """Rotating global anchor key-block columns (reading R5)."""
    if n_anchor <= 0 or n_k <= 0:
        return []
    step = n_k // n_anchor
    return sorted({(rot + t * step) % n_k for t in range(n_anchor)})


def select_row(w_row: np.ndarray, P_row: np.ndarray, k_min: int, cum_mass: float, fixed_k: int,
               anchors: Sequence[int] = ()):
    """Select the kept key blocks of one query-block row.

    Returns (kept ascending int array, info dict with m, m_p, logit gap at the
    cut and the cumulative-mass margin).
    """
    n = w_row.shape[0]
    order = rank_order(w_row)
    info = {"m_p": None, "mass_margin": math.inf}
    if fixed_k > 0:
        m = min(fixed_k, n)
    else:
        cum = np.cumsum(P_row[order])
        if cum_mass > 0:
            hit = np.nonzero(cum >= cum_mass)[0]
            m_p = int(hit[0]) + 1 if hit.size else n
        else:
            m_p = 0
        m = min(n, max(k_min, m_p))
        info["m_p"] = m_p
        if cum_mass > 0 and m >= 1:
            margins = [abs(cum[m - 1] - cum_mass)]
            if m == m_p and m >= 2:
                margins.append(abs(cum[m - 2] - cum_mass))
            info["mass_margin"] = float(min(margins))
    info["m"] = m
    if 0 < m < n:
        a, b = w_row[order[m - 1]], w_row[order[m]]
        info["gap"] = float(a - b) if np.isfinite(a) and np.isfinite(b) else math.inf
    else:
        info["gap"] = math.inf
    kept = set(int(j) for j in order[:m])
    kept.update(int(a) for a in anchors)
    return np.array(sorted(kept), dtype=np.int64), info


def select_blocks(qbar: np.ndarray, kbar: np.ndarray, n_valid: int, bq: int, bk: int, scale: float,
                  k_min: int = 0, cum_mass: float = 0.0, fixed_k: int = 0, n_anchor: int = 0,
                  anchor_rot: int = 0, with_info: bool = False):
    """Per (b, h, query block) kept key-block lists, ascending.

    qbar [B, H, n_q, d], kbar [B, H, n_k, d] are the pooled means.  Returns a
    nested list kept[b][h][i] (and, if asked, the per-row info dicts).
    """
    B, H, n_q, _ = qbar.shape
    n_k = kbar.shape[2]
    n_pad = n_q * bq
    s = valid_counts(n_pad, bk, n_valid)
    qcnt = valid_counts(n_pad, bq, n_valid)
    anchors = anchor_columns(n_k, n_anchor, anchor_rot)
    kept, infos = [], []
    for b in range(B):
        kb, ib = [], []
        for h in range(H):
            S = block_logits(qbar[b, h], kbar[b, h], scale)
            P, w = size_weighted_probs(S, s)
            kh, ih = [], []
            for i in range(n_q):
                if qcnt[i] == 0:
                    kh.append(np.zeros(0, dtype=np.int64))
                    ih.append({"m": 0, "m_p": None, "gap": math.inf, "mass_margin": math.inf})
                    continue
                row, info = select_row(w[i], P[i], k_min, cum_mass, fixed_k, anchors)
                kh.append(row)
                ih.append(info)
            kb.append(kh)
            ib.append(ih)
        kept.append(kb)
        infos.append(ib)
    return (kept, infos) if with_info else kept


def lists_to_mask(kept, n_q: int, n_k: int) -> np.ndarray:
    """Dense uint8 block mask [B, H, n_q, n_k] from kept lists."""
    B, H = len(kept), len(kept[0])
    m = np.zeros((B, H, n_q, n_k), dtype=np.uint8)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                m[b, h, i, kept[b][h][i]] = 1
    return m


# ---------------------------------------------------------------------------
# a4: block-sparse attention over the kept blocks (HVA §2 Eq. (4))
# ---------------------------------------------------------------------------

def attention_rows(q_rows: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray, scale: float):
    """Softmax attention of a few query rows over an explicit key set, fp64.

    Returns (O [r, d], LSE [r]) with LSE = ln sum_j exp(scale * q.k_j).
    An empty key set gives O = 0 and LSE = -inf (R10).
    """
    r, d = q_rows.shape
    if k_rows.shape[0] == 0:
        return np.zeros((r, d)), np.full(r, NEG_INF)
    logits = (q_rows.astype(np.float64) @ k_rows.astype(np.float64).T) * scale
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ v_rows.astype(np.float64)) / l
    return o, (m + np.log(l))[:, 0]


def _keys_of_ranges(starts: Sequence[int], length: int, n_valid: int) -> np.ndarray:
    parts = [np.arange(s, min(s + length, n_valid)) for s in starts if s < n_valid]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def block_sparse_attention(q, k, v, kept, bq: int, bk: int, n_valid: int, scale: float,
                           rows: Optional[Sequence[tuple]] = None):
    """Macro output of Eq. (4): each query block attends to its kept key blocks.

    q, k, v: [B, H, N_pad, d].  kept[b][h][i]: ascending key-block indices.
    ``rows``: optional list of (b, h, i) query blocks to evaluate (the others
    stay O = 0, LSE = -inf).  Returns (O [B, H, N_pad, d], LSE [B, H, N_pad]).
    """
    B, H, n_pad, d = q.shape
    O = np.zeros((B, H, n_pad, d))
    L = np.full((B, H, n_pad), NEG_INF)
    n_q = n_pad // bq
    todo = rows if rows is not None else [(b, h, i) for b in range(B) for h in range(H) for i in range(n_q)]
    for b, h, i in todo:
        r0, r1 = i * bq, min(i * bq + bq, n_valid)
        if r1 <= r0:
            continue
        keys = _keys_of_ranges([j * bk for j in kept[b][h][i]], bk, n_valid)
        o, lse = attention_rows(q[b, h, r0:r1], k[b, h, keys], v[b, h, keys], scale)
        O[b, h, r0:r1] = o
        L[b, h, r0:r1] = lse
    return O, L


# ---------------------------------------------------------------------------
# a5: Micro selection inside omitted blocks (HyMoR-Attn abstract)
# ---------------------------------------------------------------------------

def micro_candidates(kept_row: Sequence[int], n_k: int, bk: int, micro_keys: int, n_valid: int) -> np.ndarray:
    """Candidate 16-key tiles for a Micro row whose Macro row kept ``kept_row`` (R7)."""
    omitted = np.ones(n_k, dtype=bool)
    omitted[np.asarray(kept_row, dtype=np.int64)] = False
    per = bk // micro_keys
    tiles = np.arange(n_k * per)
    ok = omitted[tiles // per] & (tiles * micro_keys < n_valid)
    return tiles[ok]


def micro_scores(q64: np.ndarray, k16: np.ndarray, scale: float) -> np.ndarray:
    """Pooled Micro logits qbar64_r . kbar16_t * scale (R8): [..., n_r, n_t]."""
    return np.matmul(q64, np.swapaxes(k16, -1, -2)) * scale


def _micro_rows_ok(n_r: int, micro_rows: int, n_valid: int) -> np.ndarray:
    return np.arange(n_r) * micro_rows < n_valid


def select_micro_topk(q64, k16, kept, bq: int, bk: int, n_valid: int, scale: float, topk: int,
                      micro_rows: int = 64, micro_keys: int = 16, head_enable=None, with_info=False):
    """Per Micro row: the ``topk`` highest-scoring candidate tiles (R9), ascending.

    Returns tiles[b][h][r] (and per-row score gap at the cut if asked).
    """
    B, H, n_r, _ = q64.shape
    n_k = (k16.shape[2] * micro_keys) // bk
    rows_ok = _micro_rows_ok(n_r, micro_rows, n_valid)
    out, infos = [], []
    for b in range(B):
        ob, ib = [], []
        for h in range(H):
            S = micro_scores(q64[b, h], k16[b, h], scale)
            oh, ih = [], []
            for r in range(n_r):
                i = (r * micro_rows) // bq
                if not rows_ok[r] or (head_enable is not None and not head_enable[h]):
                    oh.append(np.zeros(0, dtype=np.int64))
                    ih.append(math.inf)
                    continue
                cand = micro_candidates(kept[b][h][i], n_k, bk, micro_keys, n_valid)
                sc = S[r, cand]
                order = np.lexsort((cand, -sc))
                m = min(topk, cand.size)
                sel = np.sort(cand[order[:m]])
                gap = float(sc[order[m - 1]] - sc[order[m]]) if 0 < m < cand.size else math.inf
                oh.append(sel.astype(np.int64))
                ih.append(gap)
            ob.append(oh)
            ib.append(ih)
        out.append(ob)
        infos.append(ib)
    return (out, infos) if with_info else out


def percentile_rank(q: float, M: int) -> int:
    """Nearest rank ceil(q * M), evaluated in IEEE double (R9)."""
    return int(math.ceil(float(q) * float(M)))


def select_micro_percentile(q64, k16, kept, bq: int, bk: int, n_valid: int, scale: float,
                            percentile: float, head_enable, micro_rows: int = 64, micro_keys: int = 16,
                            with_info=False):
    """Per enabled head: candidate tiles whose score is strictly above the
    nearest-rank ``percentile`` of that head's candidate scores (R9).

    Returns tiles[b][h][r] ascending (and per-head (tau, scores, candidate
    mask) if asked, for margin checks).
    """
    B, H, n_r, _ = q64.shape
    n_t = k16.shape[2]
    n_k = (n_t * micro_keys) // bk
    rows_ok = _micro_rows_ok(n_r, micro_rows, n_valid)
    out, infos = [], []
    for b in range(B):
        ob, ib = [], []
        for h in range(H):
            if not head_enable[h]:
                ob.append([np.zeros(0, dtype=np.int64) for _ in range(n_r)])
                ib.append(None)
                continue
            S = micro_scores(q64[b, h], k16[b, h], scale)
            # the head's candidate set: every (Micro row, tile) pair of R7,
            # row by row from the same rule the top-k mode uses
            cand = np.zeros((n_r, n_t), dtype=bool)
            for r in range(n_r):
                if not rows_ok[r]:
                    continue
                i = (r * micro_rows) // bq
                cand[r, micro_candidates(kept[b][h][i], n_k, bk, micro_keys, n_valid)] = True
            vals = np.sort(S[cand])
            M = vals.size
            if M == 0:
                ob.append([np.zeros(0, dtype=np.int64) for _ in range(n_r)])
                ib.append(None)
                continue
            rank = percentile_rank(percentile, M)
            rank = min(max(rank, 1), M)
            tau = vals[rank - 1]
            sel = cand & (S > tau)
            ob.append([np.nonzero(sel[r])[0].astype(np.int64) for r in range(n_r)])
            ib.append({"tau": float(tau), "M": M, "rank": rank, "S": S, "cand": cand})
        out.append(ob)
        infos.append(ib)
    return (out, infos) if with_info else out


# ---------------------------------------------------------------------------
# a6: Micro attention and exact LSE merge (HyMoR-Attn abstract)
# ---------------------------------------------------------------------------

def micro_attention(q, k, v, tiles, n_valid: int, scale: float, micro_rows: int = 64, micro_keys: int = 16,
                    rows: Optional[Sequence[tuple]] = None):
    """Attention of each 64-row Micro row over its selected 16-key tiles.

    Returns (O_mu [B, H, N_pad, d], LSE_mu [B, H, N_pad]); rows without tiles
    keep O = 0, LSE = -inf.
    """
    B, H, n_pad, d = q.shape
    O = np.zeros((B, H, n_pad, d))
    L = np.full((B, H, n_pad), NEG_INF)
    n_r = n_pad // micro_rows
    todo = rows if rows is not None else [(b, h, r) for b in range(B) for h in range(H) for r in range(n_r)]
    for b, h, r in todo:
        sel = tiles[b][h][r]
        r0, r1 = r * micro_rows, min(r * micro_rows + micro_rows, n_valid)
        if r1 <= r0 or len(sel) == 0:
            continue
        keys = _keys_of_ranges([t * micro_keys for t in sel], micro_keys, n_valid)
        o, lse = attention_rows(q[b, h, r0:r1], k[b, h, keys], v[b, h, keys], scale)
        O[b, h, r0:r1] = o
        L[b, h, r0:r1] = lse
    return O, L


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Exact merge of two attention results over disjoint key supports.

    With L = ln(e^{L_a} + e^{L_b}):  O = e^{L_a - L} O_a + e^{L_b - L} O_b.
    A side with LSE = -inf contributes nothing; both empty gives O = 0,
    LSE = -inf (R10).
    """
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    L = np.logaddexp(lse_a, lse_b)
    fin = np.isfinite(L)
    safe = np.where(fin, L, 0.0)
    wa = np.where(fin & np.isfinite(lse_a), np.exp(np.where(np.isfinite(lse_a), lse_a, 0.0) - safe), 0.0)
    wb = np.where(fin & np.isfinite(lse_b), np.exp(np.where(np.isfinite(lse_b), lse_b, 0.0) - safe), 0.0)
    O = wa[..., None] * np.asarray(o_a, dtype=np.float64) + wb[..., None] * np.asarray(o_b, dtype=np.float64)
    return O, np.where(fin, L, NEG_INF)


# ---------------------------------------------------------------------------
# Brute force on the token level (independent route for small N)
# ---------------------------------------------------------------------------

def token_mask(kept, tiles, n_pad: int, bq: int, bk: int, n_valid: int, micro_rows: int = 64,
               micro_keys: int = 16) -> np.ndarray:
    """Token-level boolean mask [B, H, N_pad, N_pad] of every (query, key) pair
    the method attends to: Macro blocks, plus Micro tiles if ``tiles`` is given."""
    B, H = len(kept), len(kept[0])
    M = np.zeros((B, H, n_pad, n_pad), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i, row in enumerate(kept[b][h]):
                for j in row:
                    M[b, h, i * bq:(i + 1) * bq, j * bk:(j + 1) * bk] = True
            if tiles is not None:
                for r, row in enumerate(tiles[b][h]):
                    for t in row:
                        M[b, h, r * micro_rows:(r + 1) * micro_rows, t * micro_keys:(t + 1) * micro_keys] = True
    M[:, :, n_valid:, :] = False
    M[:, :, :, n_valid:] = False
    return M


def masked_attention_bruteforce(q, k, v, mask: np.ndarray, scale: float):
    """Dense masked softmax attention over the full N x N logit matrix (fp64)."""
    qf, kf, vf = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    logits = np.einsum("bhnd,bhmd->bhnm", qf, kf) * scale
    logits = np.where(mask, logits, NEG_INF)
    m = logits.max(axis=-1, keepdims=True)
    has = np.isfinite(m)
    e = np.where(mask, np.exp(logits - np.where(has, m, 0.0)), 0.0)
    l = e.sum(axis=-1, keepdims=True)
    O = np.where(has, np.einsum("bhnm,bhmd->bhnd", e, vf) / np.where(has, l, 1.0), 0.0)
    L = np.where(has, m + np.log(np.where(has, l, 1.0)), NEG_INF)[..., 0]
    return O, L


# ---------------------------------------------------------------------------
# Whole path
# ---------------------------------------------------------------------------

def forward(q, k, v, w, head_enable=None, with_info: bool = False) -> Dict[str, object]:
    """Pool -> select -> Macro attention -> Micro select -> Micro attention -> merge.

    ``w`` carries the sizes and knobs (a video_inputs.Workload or anything
    with the same attribute names).  Returns a dict with the kept lists, the
    Micro tiles, the Macro (O, LSE) and the final merged (O, LSE).
    """
    n_valid, scale = w.n_valid, w.scale
    qbar = pool_block_means(q, w.bq, n_valid)
    kbar = pool_block_means(k, w.bk, n_valid)
    kept, sinfo = select_blocks(qbar, kbar, n_valid, w.bq, w.bk, scale, w.k_min, w.cum_mass, w.fixed_k,
                                w.n_anchor, w.anchor_rot, with_info=True)
    O_M, L_M = block_sparse_attention(q, k, v, kept, w.bq, w.bk, n_valid, scale)
    res = {"qbar": qbar, "kbar": kbar, "kept": kept, "select_info": sinfo, "O_macro": O_M, "LSE_macro": L_M}
    if w.micro_mode:
        q64 = pool_block_means(q, w.micro_rows, n_valid)
        k16 = pool_block_means(k, w.micro_keys, n_valid)
        if w.micro_mode == 1:
            tiles, minfo = select_micro_topk(q64, k16, kept, w.bq, w.bk, n_valid, scale, w.micro_topk,
                                             w.micro_rows, w.micro_keys, head_enable, with_info=True)
        else:
            tiles, minfo = select_micro_percentile(q64, k16, kept, w.bq, w.bk, n_valid, scale,
                                                   w.micro_percentile, head_enable, w.micro_rows,
                                                   w.micro_keys, with_info=True)
        O_mu, L_mu = micro_attention(q, k, v, tiles, n_valid, scale, w.micro_rows, w.micro_keys)
        O, L = lse_merge(O_M, L_M, O_mu, L_mu)
        res.update({"q64": q64, "k16": k16, "tiles": tiles, "micro_info": minfo, "O_micro": O_mu,
                    "LSE_micro": L_mu, "O": O, "LSE": L})
    else:
        res.update({"tiles": None, "O": O_M, "LSE": L_M})
    return res
