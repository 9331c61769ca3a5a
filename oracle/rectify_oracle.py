"""fp64 CPU oracle of pooled rectification of omitted blocks.

TEST INFRASTRUCTURE.  Like vsa_oracle, this file is the independent statement
of what the CUDA library computes, used only by the tests, the package smoke
check and the benchmark's CPU-baseline leg.  It shares no code with the CUDA
path.  Plain NumPy in float64.

Source: Rectified SpaAttn: Revisiting Attention Sparsity for Efficient Video
Generation (abstract).  Block-sparse attention biases the attention map in two
ways: the kept (critical) keys get amplified weights, because the softmax
denominator misses the mass of the omitted keys, and the omitted
(non-critical) keys lose their weight entirely.  Both are rectified with an
implicit full-attention reference built from pooled query-key interactions.
The page gives no formulas.  Readings (listed in the design notes too):

 P1 an omitted key block j of query block i stands for s_j copies of the pair
    (kbar_j, vbar_j) -- its block means over the valid keys (R1) and s_j its
    valid key count (R2): every query row q of block i gets the term
    s_j exp(scale q.kbar_j) vbar_j in the numerator and s_j exp(scale q.kbar_j)
    in the denominator (the recovered weight of the non-critical keys);
 P2 the kept keys keep their exact terms and share that denominator, so their
    weights are no longer amplified (the reallocation of the critical keys'
    weight follows from the same pooled mass; no separate factor);
 P3 the gain-aware gate of the page is not given: every omitted block with a
    valid key is rectified (in the heads where rectification is enabled);
 P4 rectification replaces the Micro repair (a layer uses one or the other);
    LSE is the natural log of the whole denominator.

Exactness: if every key block holds identical keys and identical values, the
pooled terms equal the omitted keys' exact terms and the result is dense
attention.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from .vsa_oracle import NEG_INF, pool_block_means, valid_counts

__all__ = ["rectified_rows", "rectified_attention", "forward_rectified"]


def rectified_rows(q_rows, k_kept, v_kept, kbar_om, vbar_om, s_om, scale):
    """P1/P2 for a few query rows: one softmax over the kept keys (weight 1)
    and the omitted blocks' pooled keys (weight s_j), fp64.

    Returns (O [r, d], LSE [r]); no term at all gives O = 0, LSE = -inf."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    r, d = q_rows.shape
    logits = [q_rows @ np.asarray(k_kept, dtype=np.float64).T * scale]
    values = [np.asarray(v_kept, dtype=np.float64)]
    s_om = np.asarray(s_om, dtype=np.float64)
    if s_om.size:
        logits.append(q_rows @ np.asarray(kbar_om, dtype=np.float64).T * scale + np.log(s_om)[None, :])
        values.append(np.asarray(vbar_om, dtype=np.float64))
    L = np.concatenate(logits, axis=1)
    V = np.concatenate(values, axis=0)
    if L.shape[1] == 0:
        return np.zeros((r, d)), np.full(r, NEG_INF)
    m = L.max(axis=1, keepdims=True)
    e = np.exp(L - m)
    z = e.sum(axis=1, keepdims=True)
    return (e @ V) / z, (m + np.log(z))[:, 0]


def rectified_attention(q, k, v, kept, bq: int, bk: int, n_valid: int, scale: float, rows=None):
    """Rectified block-sparse attention of one (batch, head): q, k, v
    [N_pad, d]; kept[i] the kept key blocks of query block i.  ``rows`` limits
    the work to the given query blocks.  Returns O [N_pad, d], LSE [N_pad]
    (padding rows and rows not computed: O = 0, LSE = -inf)."""
    n_pad, d = q.shape
    n_k = n_pad // bk
    kbar = pool_block_means(k[None, None], bk, n_valid)[0, 0]
    vbar = pool_block_means(v[None, None], bk, n_valid)[0, 0]
    s = valid_counts(n_pad, bk, n_valid)
    O = np.zeros((n_pad, d))
    L = np.full(n_pad, NEG_INF)
    blocks = range(n_pad // bq) if rows is None else rows
    for i in blocks:
        r0, r1 = i * bq, min((i + 1) * bq, n_valid)
        if r1 <= r0:
            continue
        kept_i = sorted(int(j) for j in kept[i])
        keys = np.concatenate([np.arange(j * bk, min((j + 1) * bk, n_valid)) for j in kept_i]) if kept_i else \
            np.zeros(0, dtype=np.int64)
        om = [j for j in range(n_k) if j not in set(kept_i) and s[j] > 0]
        o, lse = rectified_rows(q[r0:r1], k[keys], v[keys], kbar[om], vbar[om], s[om], scale)
        O[r0:r1] = o
        L[r0:r1] = lse
    return O, L


def forward_rectified(q, k, v, w, head_enable: Optional[Sequence[int]] = None) -> Dict[str, object]:
    """Pooling, selection (the path's rule) and rectified attention for every
    (batch, head) of a workload; heads with head_enable[h] == 0 get the plain
    block-sparse attention."""
    from .vsa_oracle import block_sparse_attention, select_blocks
    B, H, n_pad, d = q.shape
    O = np.zeros((B, H, n_pad, d))
    L = np.full((B, H, n_pad), NEG_INF)
    kept_all = []
    for b in range(B):
        for h in range(H):
            qb = pool_block_means(q[b:b + 1, h:h + 1], w.bq, w.n_valid)
            kb = pool_block_means(k[b:b + 1, h:h + 1], w.bk, w.n_valid)
            kept = select_blocks(qb, kb, w.n_valid, w.bq, w.bk, w.scale, w.k_min, w.cum_mass, w.fixed_k,
                                 w.n_anchor, w.anchor_rot)[0][0]
            kept_all.append(kept)
            if head_enable is None or head_enable[h]:
                O[b, h], L[b, h] = rectified_attention(q[b, h], k[b, h], v[b, h], kept, w.bq, w.bk, w.n_valid,
                                                       w.scale)
            else:
                o, l = block_sparse_attention(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                                              [[kept]], w.bq, w.bk, w.n_valid, w.scale)
                O[b, h], L[b, h] = o[0, 0], l[0, 0]
    return {"O": O, "LSE": L, "kept": kept_all}
