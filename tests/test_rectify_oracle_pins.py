"""Pins of the pooled-rectification oracle (Rectified SpaAttn abstract;
readings P1-P4 in oracle/rectify_oracle.py), each against something other
than the oracle itself: a hand-worked example, dense attention when every
key block is uniform (where pooling is exact), and an explicit duplicated-key
attention in which an omitted block is s_j real copies of its mean key/value.
"""
import os

import numpy as np
import pytest

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rectify_hand.txt")


def _dense(q, k, v, n_valid, scale):
    """Plain softmax attention of every valid row over every valid key."""
    L = q[:n_valid] @ k[:n_valid].T * scale
    m = L.max(axis=1, keepdims=True)
    e = np.exp(L - m)
    return (e @ v[:n_valid]) / e.sum(axis=1, keepdims=True), (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]


def test_hand_worked_example():
    q = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [0.0, 0.0]])
    k = np.array([[0.0, 0.0], [1.0, 0.0], [2.0, 0.0], [5.0, 5.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [9.0, 9.0]])
    O, L = orc.rectified_attention(q, k, v, [[1], [0]], 2, 2, 3, 1.0)
    rows = [l.split() for l in open(GOLDEN) if l[0].isdigit()]
    assert len(rows) == 3
    for r, _, o0, o1, lse in rows:
        r = int(r)
        assert np.allclose(O[r], [float(o0), float(o1)], rtol=0, atol=1e-14)
        assert abs(L[r] - float(lse)) < 1e-14
    assert np.all(O[3] == 0) and L[3] == -np.inf


@pytest.mark.parametrize("seed,n_valid", [(0, 250), (1, 256), (2, 193)])
def test_uniform_blocks_give_dense_attention(seed, n_valid):
    """Identical keys and values inside every key block: each pooled term is
    exactly its block's keys, so rectified attention equals dense attention
    whatever was kept."""
    rng = np.random.default_rng(seed)
    n_pad, bq, bk, d = 256, 32, 32, 8
    nb = n_pad // bk
    kb, vb = rng.standard_normal((nb, d)), rng.standard_normal((nb, d))
    k, v = np.repeat(kb, bk, axis=0), np.repeat(vb, bk, axis=0)
    q = rng.standard_normal((n_pad, d))
    kept = [sorted(rng.choice(nb, size=int(rng.integers(0, nb + 1)), replace=False).tolist())
            for _ in range(n_pad // bq)]
    kept[0], kept[1] = [], list(range(nb))
    O, L = orc.rectified_attention(q, k, v, kept, bq, bk, n_valid, 0.4)
    Od, Ld = _dense(q, k, v, n_valid, 0.4)
    assert np.allclose(O[:n_valid], Od, rtol=0, atol=1e-12)
    assert np.allclose(L[:n_valid], Ld, rtol=0, atol=1e-12)
    assert np.all(O[n_valid:] == 0) and np.all(L[n_valid:] == -np.inf)


def test_every_block_kept_is_plain_block_sparse():
    rng = np.random.default_rng(4)
    n_pad, bq, bk, d, n_valid = 192, 64, 32, 16, 180
    q, k, v = (rng.standard_normal((n_pad, d)) for _ in range(3))
    kept = [list(range(n_pad // bk))] * (n_pad // bq)
    O, L = orc.rectified_attention(q, k, v, kept, bq, bk, n_valid, 0.25)
    Ob, Lb = orc.block_sparse_attention(q[None, None], k[None, None], v[None, None], [[kept]], bq, bk, n_valid, 0.25)
    assert np.allclose(O, Ob[0, 0], rtol=0, atol=1e-12)
    assert np.array_equal(np.isfinite(L), np.isfinite(Lb[0, 0]))
    assert np.allclose(L[:n_valid], Lb[0, 0, :n_valid], rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [5, 6])
def test_equals_attention_over_duplicated_block_means(seed):
    """An omitted block as s_j explicit copies of (kbar_j, vbar_j) (a ragged
    last block has fewer copies): plain attention over kept keys plus the
    copies must equal the weighted-softmax form."""
    rng = np.random.default_rng(seed)
    n_pad, bq, bk, d, n_valid = 160, 32, 32, 8, 150
    q, k, v = (rng.standard_normal((n_pad, d)) for _ in range(3))
    nb = n_pad // bk
    kept = [sorted(rng.choice(nb, size=int(rng.integers(0, nb)), replace=False).tolist()) for _ in range(n_pad // bq)]
    O, L = orc.rectified_attention(q, k, v, kept, bq, bk, n_valid, 0.3)
    for i, ki in enumerate(kept):
        r0, r1 = i * bq, min((i + 1) * bq, n_valid)
        keys, vals = [], []
        for j in range(nb):
            lo, hi = j * bk, min((j + 1) * bk, n_valid)
            if hi <= lo:
                continue
            if j in ki:
                keys.append(k[lo:hi])
                vals.append(v[lo:hi])
            else:
                keys.append(np.repeat(k[lo:hi].mean(axis=0)[None], hi - lo, axis=0))
                vals.append(np.repeat(v[lo:hi].mean(axis=0)[None], hi - lo, axis=0))
        o, l = orc.attention_rows(q[r0:r1], np.concatenate(keys), np.concatenate(vals), 0.3)
        assert np.allclose(O[r0:r1], o, rtol=0, atol=1e-12)
        assert np.allclose(L[r0:r1], l, rtol=0, atol=1e-12)


def test_rectification_moves_toward_dense_on_smooth_blocks():
    """Keys that vary little inside a block: rectified attention is much
    closer to dense attention than the plain block-sparse output."""
    rng = np.random.default_rng(8)
    n_pad, bq, bk, d = 256, 32, 32, 16
    nb = n_pad // bk
    kb, vb = rng.standard_normal((nb, d)), rng.standard_normal((nb, d))
    k = np.repeat(kb, bk, axis=0) + 0.05 * rng.standard_normal((n_pad, d))
    v = np.repeat(vb, bk, axis=0) + 0.05 * rng.standard_normal((n_pad, d))
    q = rng.standard_normal((n_pad, d))
    kept = [sorted(rng.choice(nb, size=3, replace=False).tolist()) for _ in range(n_pad // bq)]
    O, _ = orc.rectified_attention(q, k, v, kept, bq, bk, n_pad, 0.5)
    Ob, _ = orc.block_sparse_attention(q[None, None], k[None, None], v[None, None], [[kept]], bq, bk, n_pad, 0.5)
    Od, _ = _dense(q, k, v, n_pad, 0.5)
    assert np.linalg.norm(O - Od) < 0.2 * np.linalg.norm(Ob[0, 0] - Od)
