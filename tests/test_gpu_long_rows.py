"""Selection rows longer than 1024 key blocks (one CTA per row instead of one
warp): a layer of 1536 key blocks of 64 keys (n_pad = 98,304, 64-row query
blocks), in fixed-k mode with anchors and in Top-p mode with a Min-kc floor,
against the fp64 oracle with the selection rule of gpu_helpers; the explicit
mask path on the same rows; Micro selection (per-head percentile) over the
same lists; and attention over the long lists on sampled rows.  Sources:
HyperVAttention §2 Eq. (2)-(4), App. A.1 (Min-kc); LVSA abstract (anchors);
HyMoR-Attn abstract (Micro tiles in omitted blocks).
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import Workload, make_qkv

from gpu_helpers import GAP, assert_close_rows, compare_selection, oracle_select_per_head, to_dev

pytestmark = pytest.mark.gpu

BASE = Workload("long1536", 1, 2, 128, (24, 32, 127), 64, 64, seed=11, generator="locality", field_scale=0.8,
                n_pad_fixed=98_304)
RULES = {
    "fixed": dict(fixed_k=230, n_anchor=2, anchor_rot=5),
    "top_p": dict(cum_mass=0.9, k_min=16),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    torch.cuda.init()
    yield
    assert vsa.read_device_status() == 0


@pytest.fixture(scope="module")
def qkv():
    return make_qkv(BASE)


@pytest.mark.parametrize("rule", list(RULES))
def test_selection_of_1536_key_blocks(qkv, rule):
    w = dataclasses.replace(BASE, **RULES[rule])
    assert w.n_k == 1536 and w.n_valid < w.n_pad
    q, k, v = qkv
    H = q.shape[1]
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qp = torch.empty(w.B, H, w.n_q, w.d, device="cuda")
    kp = torch.empty(w.B, H, w.n_k, w.d, device="cuda")
    q64 = torch.empty(w.B, H, w.n_pad // 64, w.d, device="cuda")
    k16 = torch.empty(w.B, H, w.n_pad // 16, w.d, device="cuda")
    vsa.pool_qk(dq, dk, shape, w.bq, w.bk, qp, kp, q64, k16)
    counts = torch.empty(w.B, H, w.n_q, dtype=torch.int32, device="cuda")
    idx = torch.full((w.B, H, w.n_q, w.n_k), -3, dtype=torch.int32, device="cuda")
    mask = torch.empty(w.B, H, w.n_q, w.n_k, dtype=torch.uint8, device="cuda")
    vsa.select_blocks(qp, kp, shape, w.bq, w.bk, w.scale,
                      vsa.SelectParams(w.k_min, w.cum_mass, w.fixed_k, w.n_anchor, w.anchor_rot), counts, idx, mask)
    assert vsa.read_device_status() == 0
    c, ix, mk = counts.cpu().numpy(), idx.cpu().numpy(), mask.cpu().numpy()
    kept, info, logw, probs, _, _ = oracle_select_per_head(q, k, w)
    n_exact, n_near, n_1e3 = compare_selection(c, ix, kept, info, logw, probs, w, gpu_mask=mk)
    print(f"\n{rule}: rows bit-exact {n_exact}, near-tie valid {n_near} (gap < 1e-3: {n_1e3})")
    n_q_valid = -(-w.n_valid // w.bq)
    assert np.all(c[:, :, n_q_valid:] == 0)
    # the mask path gives back the same lists
    c2 = torch.empty_like(counts)
    ix2 = torch.full_like(idx, -3)
    vsa.mask_to_lists(mask, shape, w.bq, w.bk, c2, ix2)
    assert vsa.read_device_status() == 0
    assert torch.equal(c2, counts)
    valid = torch.arange(w.n_k, device="cuda").view(1, 1, 1, -1) < counts.unsqueeze(-1)
    assert torch.equal(ix2[valid], idx[valid])

    if rule != "fixed":
        return
    # Micro selection (percentile, head 0 only) over lists of 1536 blocks
    flags = [1, 0]
    cap = w.n_pad // 16
    mc = torch.empty(w.B, H, w.n_pad // 64, dtype=torch.int32, device="cuda")
    mi = torch.empty(w.B, H, w.n_pad // 64, cap, dtype=torch.int32, device="cuda")
    ws = torch.empty(vsa.select_micro_workspace_bytes(shape, 2, 0, 0.99, flags, cap), dtype=torch.uint8,
                     device="cuda")
    vsa.select_micro(q64, k16, counts, idx, shape, w.bq, w.bk, w.scale, 2, 0, 0.99, flags, cap, mc, mi, ws)
    assert vsa.read_device_status() == 0
    mcn, min_ = mc.cpu().numpy(), mi.cpu().numpy()
    assert np.all(mcn[0, 1] == 0)
    gk = [[[ix[0, 0, i, :c[0, 0, i]] for i in range(w.n_q)]]]     # the GPU's Macro lists of head 0
    same = all(np.array_equal(gk[0][0][i], kept[0][0][i]) for i in range(w.n_q))
    q64o = orc.pool_block_means(q[:, :1], 64, w.n_valid)
    k16o = orc.pool_block_means(k[:, :1], 16, w.n_valid)
    if same:
        tiles, minfo = orc.select_micro_percentile(q64o, k16o, kept, w.bq, w.bk, w.n_valid, w.scale, 0.99,
                                                   np.array([1]), with_info=True)
        inf = minfo[0][0]
        far = inf["cand"] & (np.abs(inf["S"] - inf["tau"]) >= GAP)
        sel_o = np.zeros_like(far)
        for r, t in enumerate(tiles[0][0]):
            sel_o[r, t] = True
        sel_g = np.zeros_like(far)
        for r in range(far.shape[0]):
            sel_g[r, min_[0, 0, r, :mcn[0, 0, r]]] = True
        assert np.array_equal(sel_g[far], sel_o[far])
        assert not np.any(sel_g & ~inf["cand"])
        print(f"  Micro: {int(sel_g.sum())} tiles, {int(far.sum())} candidates compared exactly")
    # attention over the oracle's long lists (64-row lists of 64-key blocks), sampled rows
    n_l = w.n_q
    cnt = np.zeros((1, H, n_l), dtype=np.int32)
    lst = np.zeros((1, H, n_l, w.n_k), dtype=np.int32)
    for h in range(H):
        for i in range(n_l):
            row = kept[0][h][i]
            cnt[0, h, i] = len(row)
            lst[0, h, i, :len(row)] = row
    o = torch.empty(w.B, H, w.n_pad, w.d, device="cuda")
    lse = torch.empty(w.B, H, w.n_pad, device="cuda")
    vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, torch.from_numpy(cnt).cuda(), torch.from_numpy(lst).cuda(),
                         w.n_k, w.scale, o, lse)
    assert vsa.read_device_status() == 0
    rows = [(0, h, i) for h in range(H) for i in (0, 1, 700, n_q_valid - 1, w.n_q - 1)]
    O, L = orc.block_sparse_attention(q, k, v, kept, w.bq, w.bk, w.n_valid, w.scale, rows=rows)
    assert_close_rows(o.cpu().numpy(), lse.cpu().numpy(), O, L, [(b, h, i * w.bq, (i + 1) * w.bq) for b, h, i in rows])
