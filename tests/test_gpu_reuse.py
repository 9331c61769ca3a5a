"""GPU parity of cross-step mask reuse: a step that reuses the selection
attends the new step's Q, K, V with the lists selected at an earlier step --
Macro and Micro lists alike -- and equals the oracle's attention with exactly
those lists."""
import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv, micro_heads, round_to_bf16

from gpu_helpers import assert_close_rows, to_dev
from test_gpu_rectify import _check_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    yield
    assert vsa.read_device_status() == 0


def _next_step(x, seed, drift=0.3):
    """A later denoising step: the same tensor plus seeded noise, in bf16."""
    rng = np.random.default_rng(seed)
    return round_to_bf16((x + drift * rng.standard_normal(x.shape).astype(np.float32)).astype(np.float32))


def test_reused_lists_attend_the_new_step():
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    heads = micro_heads(w)
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    with pytest.raises(ValueError):
        run(to_dev(q), to_dev(k), to_dev(v), reuse_selection=True)
    run(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    lists = {n: run.buf[n].clone() for n in ("counts", "idx", "m_counts", "m_idx")}
    q2, k2, v2 = (_next_step(x, s) for x, s in ((q, 11), (k, 12), (v, 13)))
    out = run(to_dev(q2), to_dev(k2), to_dev(v2), reuse_selection=True)
    torch.cuda.synchronize()
    assert vsa.read_device_status() == 0
    for n, t in lists.items():
        assert torch.equal(run.buf[n], t), n
    counts, idx = lists["counts"].cpu().numpy(), lists["idx"].cpu().numpy()
    mc, mi = lists["m_counts"].cpu().numpy(), lists["m_idx"].cpu().numpy()
    kept = [[[idx[0, h, i, :counts[0, h, i]] for i in range(w.n_pad // w.bq)] for h in range(w.H)]]
    tiles = [[[mi[0, h, r, :mc[0, h, r]] if heads[h] else np.zeros(0, dtype=np.int64)
               for r in range(w.n_pad // 64)] for h in range(w.H)]]
    O_mac, L_mac = orc.block_sparse_attention(q2, k2, v2, kept, w.bq, w.bk, w.n_valid, w.scale)
    O_mu, L_mu = orc.micro_attention(q2, k2, v2, tiles, w.n_valid, w.scale)
    O, L = orc.lse_merge(O_mac, L_mac, O_mu, L_mu)
    assert_close_rows(out["o"].float().cpu().numpy(), out["lse"].cpu().numpy(), O, L,
                      [(0, h, 0, w.n_pad) for h in range(w.H)], bf16_out=True)
    # and the fresh selection on the new step differs from the reused one somewhere
    fresh = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))(to_dev(q2), to_dev(k2), to_dev(v2))
    torch.cuda.synchronize()
    assert not (torch.equal(fresh["idx"], lists["idx"]) and torch.equal(fresh["m_idx"], lists["m_idx"]))


def test_reuse_with_rectification_repools_the_new_step():
    """Under rectification the reused lists name the omitted blocks, but their
    pooled keys and values are those of the new step."""
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    cfg = vsa.PathConfig.from_workload(w)
    cfg.micro_mode = 0
    cfg.rectify = True
    run = vsa.SparseVideoAttention(cfg)
    run(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    lists = (run.buf["counts"].clone(), run.buf["idx"].clone())
    q2, k2, v2 = (_next_step(x, s) for x, s in ((q, 21), (k, 22), (v, 23)))
    out = run(to_dev(q2), to_dev(k2), to_dev(v2), reuse_selection=True)
    torch.cuda.synchronize()
    assert vsa.read_device_status() == 0
    assert torch.equal(out["counts"], lists[0]) and torch.equal(out["idx"], lists[1])
    # the rectification tests' comparison (tolerance derived from the bf16 pooled rows)
    for h in range(w.H):
        _check_rows(w, out, q2, k2, v2, h, list(range(w.n_pad // w.bq)), True)
