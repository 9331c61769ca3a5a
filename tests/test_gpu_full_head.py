"""Complete-head parity at full size: every query block and every Micro row of
one head of the large layers, element by element against the fp64 oracle.

Two comparisons per layer, both on the launch configuration of the whole path
(all heads of the layer in one call, as the benchmark runs it):

  * the path as it runs (GPU pooling, selection, Macro pass, Micro selection,
    Micro pass + merge): the head's kept lists checked row by row with the
    selection rule of gpu_helpers (bit-exact where the cut is decided, a
    valid answer at near ties), the Micro tiles exact away from the
    percentile threshold and valid near it, and O / LSE of every query block
    whose Macro list and both Micro lists equal the oracle's;
  * the same attention passes fed the ORACLE's lists for that head (the
    path's reuse-selection mode: no pooling or selection runs): O / LSE of
    every row of the head, with no exclusion.

Sources: HyperVAttention §2 Eq. (2)-(4) (selection and attention over the
kept blocks), App. A.1 (Min-kc); HyMoR-Attn abstract (Micro residual, exact
LSE merge); LVSA abstract (rotating anchors).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv, micro_heads

from gpu_helpers import GAP, assert_close_rows, compare_selection, oracle_select_per_head, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    torch.cuda.init()
    yield
    assert vsa.read_device_status() == 0


def _micro_check(mc, mi, tiles, inf):
    """Micro tiles of one head: exact where the oracle score is at least GAP
    from tau, and only candidates, with a count that differs by no more than
    the near-tau tiles.  Returns (tiles compared exactly, near-tau tiles)."""
    far = inf["cand"] & (np.abs(inf["S"] - inf["tau"]) >= GAP)
    sel_o = np.zeros_like(far)
    for r, t in enumerate(tiles):
        sel_o[r, t] = True
    sel_g = np.zeros_like(far)
    for r in range(far.shape[0]):
        row = mi[r, :mc[r]]
        assert np.all(np.diff(row) > 0), (r, "not ascending")
        sel_g[r, row] = True
    assert np.array_equal(sel_g[far], sel_o[far])
    assert not np.any(sel_g & ~inf["cand"])
    near = inf["cand"] & ~far
    # a near-tau tile may go either way, and nothing else may differ
    assert np.array_equal(sel_g & ~near, sel_o & ~near)
    return int(far.sum()), int(near.sum())


def _head_oracle(w, q, k, v, h, micro_flag):
    """Oracle lists and output of head h (inputs of all heads given)."""
    qh, kh, vh = q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1]
    kept, info, logw, probs, _, _ = oracle_select_per_head(qh, kh, w)
    res = {"kept": kept, "info": info, "logw": logw, "probs": probs}
    O_M, L_M = orc.block_sparse_attention(qh, kh, vh, kept, w.bq, w.bk, w.n_valid, w.scale)
    res["O_macro"], res["L_macro"] = O_M, L_M
    if micro_flag:
        q64 = orc.pool_block_means(qh, 64, w.n_valid)
        k16 = orc.pool_block_means(kh, 16, w.n_valid)
        tiles, minfo = orc.select_micro_percentile(q64, k16, kept, w.bq, w.bk, w.n_valid, w.scale,
                                                   w.micro_percentile, np.array([1], dtype=np.uint8),
                                                   with_info=True)
        O_u, L_u = orc.micro_attention(qh, kh, vh, tiles, w.n_valid, w.scale)
        O, L = orc.lse_merge(O_M, L_M, O_u, L_u)
        res.update({"tiles": tiles, "micro_info": minfo, "O": O, "L": L})
    else:
        res.update({"tiles": None, "O": O_M, "L": L_M})
    return res


def _lists_into(run, h, kept, tiles, w):
    """Write head h's oracle lists into the path's list buffers."""
    b = run.buf
    n_q, n_k = w.n_pad // w.bq, w.n_pad // w.bk
    counts = np.zeros(n_q, dtype=np.int32)
    idx = np.zeros((n_q, n_k), dtype=np.int32)
    for i, row in enumerate(kept[0][0]):
        counts[i] = len(row)
        idx[i, :len(row)] = row
    b["counts"][0, h] = torch.from_numpy(counts)
    b["idx"][0, h] = torch.from_numpy(idx)
    if tiles is not None:
        cap = b["m_idx"].shape[-1]
        n_r = w.n_pad // 64
        mc = np.zeros(n_r, dtype=np.int32)
        mi = np.zeros((n_r, cap), dtype=np.int32)
        for r, row in enumerate(tiles[0][0]):
            assert len(row) <= cap
            mc[r] = len(row)
            mi[r, :len(row)] = row
        b["m_counts"][0, h] = torch.from_numpy(mc)
        b["m_idx"][0, h] = torch.from_numpy(mi)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name,heads,h", [("hunyuan", None, None), ("wan14b", (0, 4), 1), ("wan13b", None, 3)])
def test_complete_head(name, heads, h):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    flags = micro_heads(w)[:H] if w.micro_mode else None
    if h is None:                                   # the first Micro head of the layer
        h = int(np.nonzero(flags)[0][0])
    micro_flag = bool(flags is not None and flags[h])
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, flags))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    del_dev = lambda t: t[0, h].cpu().numpy()
    out = run(dq, dk, dv)
    assert vsa.read_device_status() == 0
    counts, idx = del_dev(out["counts"])[None, None], del_dev(out["idx"])[None, None]
    O_path = out["o"][0, h].float().cpu().numpy()[None, None]
    L_path = out["lse"][0, h].cpu().numpy()[None, None]
    if micro_flag:
        mc, mi = del_dev(out["m_counts"]), del_dev(out["m_idx"])

    ref = _head_oracle(w, q, k, v, h, micro_flag)
    n_exact, n_near, n_1e3 = compare_selection(counts, idx, ref["kept"], ref["info"], ref["logw"], ref["probs"], w)
    print(f"\n{name} head {h}: {n_exact + n_near} query blocks, selection bit-exact {n_exact}, near-tie valid {n_near}"
          f" (gap < 1e-3: {n_1e3})")
    same = [i for i in range(w.n_q) if np.array_equal(idx[0, 0, i, :counts[0, 0, i]], ref["kept"][0][0][i])]
    if micro_flag:
        n_far, n_neartau = _micro_check(mc, mi, ref["tiles"][0][0], ref["micro_info"][0][0])
        n_sel = int(mc.sum())
        print(f"  Micro: {w.n_pad // 64} rows, {n_sel} tiles selected; {n_far} candidate tiles compared exactly,"
              f" {n_neartau} within {GAP} of tau")
        same = [i for i in same
                if all(np.array_equal(mi[r, :mc[r]], ref["tiles"][0][0][r]) for r in (2 * i, 2 * i + 1))]
    assert len(same) >= 0.9 * w.n_q, (len(same), w.n_q)
    worst = assert_close_rows(O_path, L_path, ref["O"], ref["L"],
                              [(0, 0, i * w.bq, (i + 1) * w.bq) for i in same], bf16_out=True)
    print(f"  whole path: {len(same)} of {w.n_q} query blocks compared, worst |dO| {worst[0]:.2e}, "
          f"|dLSE| {worst[1]:.2e}")

    # the attention passes on the oracle's lists: every row of the head
    _lists_into(run, h, ref["kept"], ref["tiles"], w)
    out = run(dq, dk, dv, reuse_selection=True)
    assert vsa.read_device_status() == 0
    O_all = out["o"][0, h].float().cpu().numpy()[None, None]
    L_all = out["lse"][0, h].cpu().numpy()[None, None]
    worst = assert_close_rows(O_all, L_all, ref["O"], ref["L"], [(0, 0, 0, w.n_pad)], bf16_out=True)
    print(f"  oracle lists: all {w.n_pad} rows, worst |dO| {worst[0]:.2e}, |dLSE| {worst[1]:.2e}")
