"""GPU parity of pooled rectification of omitted blocks (Rectified SpaAttn
abstract; readings P1-P4 of the rectification oracle) through the C ABI.

The kernel multiplies bf16 operands, so the pooled keys and values enter it
rounded to bf16.  Each pooled logit is then off by at most
delta = scale * max_j |q . (kbar_j - kbar_j^gpu)| for the row, computed here
from the GPU's own pooled rows; LSE moves by at most delta and every softmax
weight by a factor within exp(+-2 delta).  The comparison adds exactly that to
the attention tolerances: |dLSE| <= LSE_TOL + delta and
|dO| <= O_TOL + (exp(2 delta) - 1) max|value| + max|vbar - vbar^gpu|, plus
half a bf16 ulp of O for the bf16 output.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv, sweep_points

from gpu_helpers import LSE_TOL, O_TOL, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    yield
    assert vsa.read_device_status() == 0


def _workload(name):
    if name.startswith("sweep"):
        return [w for _, w in sweep_points() if w.name == name][0]
    return WORKLOADS[name]


@pytest.mark.parametrize("name,heads", [("tiny", None), ("wan13b", (0, 2)), ("sweep-64x128-8pct", (0, 1))])
def test_pool_kv_bf16_is_the_rounded_block_mean(name, heads):
    w = _workload(name)
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    n_k = w.n_pad // w.bk
    rows = -(-n_k // 128) * 128 + 128
    kb = torch.full((w.B, H, rows, w.d), 7.0, device="cuda", dtype=torch.bfloat16)
    vb = torch.full_like(kb, 7.0)
    vsa.pool_kv_bf16(to_dev(k), to_dev(v), shape, w.bk, kb, vb)
    assert vsa.read_device_status() == 0
    for x, xb in ((k, kb), (v, vb)):
        want = orc.pool_block_means(x, w.bk, w.n_valid)
        got = xb.float().cpu().numpy()[:, :, :n_k]
        # fp32 sum and one rounding to bf16: within one bf16 ulp of the exact mean
        assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)
        assert np.all(xb.float().cpu().numpy()[:, :, n_k:] == 0)


def _run(w, q, k, v, flags):
    cfg = vsa.PathConfig.from_workload(w)
    cfg.micro_mode = 0
    cfg.rectify = True
    cfg.rectify_heads = flags
    run = vsa.SparseVideoAttention(cfg)
    b = run(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert vsa.read_device_status() == 0
    return b


def _check_rows(w, b, q, k, v, h, blocks, rectified):
    counts = b["counts"][0, h].cpu().numpy()
    idx = b["idx"][0, h].cpu().numpy()
    kept = [idx[i, :counts[i]] for i in range(w.n_pad // w.bq)]
    og = b["o"][0, h].float().cpu().numpy()
    lg = b["lse"][0, h].cpu().numpy()
    qh, kh, vh = (x[0, h].astype(np.float64) for x in (q, k, v))
    worst = 0.0
    if rectified:
        O, L = orc.rectified_attention(qh, kh, vh, kept, w.bq, w.bk, w.n_valid, w.scale, rows=blocks)
        kbar = orc.pool_block_means(k[:, h:h + 1], w.bk, w.n_valid)[0, 0]
        vbar = orc.pool_block_means(v[:, h:h + 1], w.bk, w.n_valid)[0, 0]
        n_k = kbar.shape[0]
        kg = b["k_bar"][0, h].float().cpu().numpy()[:n_k]
        vg = b["v_bar"][0, h].float().cpu().numpy()[:n_k]
    else:
        O, L = orc.block_sparse_attention(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], [[kept]], w.bq, w.bk,
                                          w.n_valid, w.scale, rows=[(0, 0, i) for i in blocks])
        O, L = O[0, 0], L[0, 0]
    for i in blocks:
        r0, r1 = i * w.bq, min((i + 1) * w.bq, w.n_pad)
        rv = min(r1, w.n_valid)
        if rv <= r0:  # a query block of padding rows only
            assert np.all(og[r0:r1] == 0) and np.all(~np.isfinite(lg[r0:r1]))
            continue
        if rectified and rv > r0:
            om = [j for j in range(n_k) if j not in set(kept[i].tolist())]
            dl = np.abs(qh[r0:rv] @ (kbar[om] - kg[om]).T) * w.scale if om else np.zeros((rv - r0, 1))
            delta = dl.max(axis=1)
            ev = float(np.abs(vbar[om] - vg[om]).max()) if om else 0.0
            vmax = max(float(np.abs(vh[:w.n_valid]).max()), float(np.abs(vbar).max()))
        else:
            delta = np.zeros(max(0, rv - r0))
            ev, vmax = 0.0, 0.0
        lref, lgpu = L[r0:r1], lg[r0:r1]
        assert np.array_equal(np.isfinite(lref), np.isfinite(lgpu)), (h, i)
        fin = np.isfinite(lref[:rv - r0])
        d_l = np.abs(lgpu[:rv - r0] - lref[:rv - r0])
        assert np.all(d_l[fin] <= LSE_TOL + delta[fin]), (h, i, float((d_l - delta).max()))
        allow = np.abs(O[r0:rv]) * 2.0 ** -8 + O_TOL + ((np.exp(2 * delta) - 1) * vmax + ev)[:, None]
        d_o = np.abs(og[r0:rv] - O[r0:rv])
        assert np.all(d_o <= allow), (h, i, float((d_o - allow).max()))
        assert np.all(og[rv:r1] == 0) and np.all(~np.isfinite(lgpu[rv - r0:]))
        worst = max(worst, float(d_o.max()) if d_o.size else 0.0)
    return worst


@pytest.mark.parametrize("name,heads,n_blocks,flags", [
    ("tiny", None, None, None),
    ("wan13b", (0, 2), 6, None),
    ("hunyuan", (0, 2), 4, (1, 0)),          # one rectified head, one plain head
    ("sweep-64x128-8pct", (0, 1), 6, None),  # 64-row query blocks: two lists per tile
])
def test_rectified_path_matches_the_oracle(name, heads, n_blocks, flags):
    w = _workload(name)
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    wl = dataclasses.replace(w, H=H)
    b = _run(wl, q, k, v, flags)
    n_q = w.n_pad // w.bq
    rng = np.random.default_rng(3)
    for h in range(H):
        if n_blocks is None:
            blocks = list(range(n_q))
        else:
            last = (w.n_valid - 1) // w.bq
            blocks = sorted({0, last, n_q - 1} | set(rng.choice(n_q, size=n_blocks, replace=False).tolist()))
        worst = _check_rows(wl, b, q, k, v, h, blocks, flags is None or bool(flags[h]))
        print(f"\n{name} head {h}: worst |dO| {worst:.2e}")


def test_rectify_with_nothing_omitted_is_the_plain_path():
    """Every block kept: the pooled pass adds nothing and the merged output is
    the plain block-sparse output bit for bit."""
    w = dataclasses.replace(WORKLOADS["wan13b"], cum_mass=0.0, k_min=0, fixed_k=WORKLOADS["wan13b"].n_pad // 128)
    q, k, v = make_qkv(w, heads=(0, 2))
    wl = dataclasses.replace(w, H=2)
    b = _run(wl, q, k, v, None)
    o_r, l_r = b["o"].clone(), b["lse"].clone()
    cfg = vsa.PathConfig.from_workload(wl)
    cfg.micro_mode = 0
    plain = vsa.SparseVideoAttention(cfg)(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert torch.equal(o_r, plain["o"]) and torch.equal(l_r, plain["lse"])


def test_uniform_blocks_give_dense_attention_on_the_gpu():
    """Keys and values identical inside every key block: the pooled means are
    exact in bf16 and the rectified output is dense attention (the same kernel
    with every block kept)."""
    w = dataclasses.replace(WORKLOADS["wan13b"], cum_mass=0.0, k_min=0, fixed_k=20)
    q, k, v = make_qkv(w, heads=(0, 1))
    nb = w.n_pad // w.bk
    k = np.repeat(k[:, :, ::w.bk][:, :, :nb], w.bk, axis=2)
    v = np.repeat(v[:, :, ::w.bk][:, :, :nb], w.bk, axis=2)
    k[:, :, w.n_valid:] = 0
    v[:, :, w.n_valid:] = 0
    wl = dataclasses.replace(w, H=1)
    b = _run(wl, q, k, v, None)
    o_r = b["o"].float().cpu().numpy()
    dense = vsa.SparseVideoAttention(vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale, fixed_k=nb))
    o_d = dense(to_dev(q), to_dev(k), to_dev(v))["o"].float().cpu().numpy()
    assert np.abs(o_r - o_d)[:, :, :w.n_valid].max() <= 2 * O_TOL
