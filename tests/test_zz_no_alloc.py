"""The allocation-free Micro selection gives the same lists as the workspace one.

vsa_select_micro_noalloc serves callers that cannot allocate device memory of
their own (an engine plugin that is handed no workspace, a service whose
device memory belongs to another allocator): it keeps its scratch in one fixed
array that the library reserves on each GPU.  This file checks, through the C
ABI, that its Micro lists equal those of vsa_select_micro (integer outputs,
compared bit-exactly as in the other tests) on two calls in a row -- the
second call reuses the fixed array the first one left behind -- and that a
problem too large for the fixed array is refused.  It is collected last and
passes both alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
from video_inputs import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    yield
    assert vsa.read_device_status() == 0


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(torch.bfloat16).contiguous()


def _pooled_and_lists(w, H):
    """Pooled means and Macro lists of the first H heads, all from libvsa."""
    q, k, _ = make_qkv(w, heads=(0, H))
    shape = vsa.Shape(w.B, H, w.n_valid, w.n_pad, w.d)
    dq, dk = _dev(q), _dev(k)
    n_q, n_k = w.n_pad // w.bq, w.n_pad // w.bk
    f = lambda n: torch.empty(w.B, H, w.n_pad // n, w.d, device="cuda")
    qp, kp, q64, k16 = f(w.bq), f(w.bk), f(64), f(16)
    vsa.pool_qk(dq, dk, shape, w.bq, w.bk, qp, kp, q64, k16)
    counts = torch.empty(w.B, H, n_q, dtype=torch.int32, device="cuda")
    idx = torch.empty(w.B, H, n_q, n_k, dtype=torch.int32, device="cuda")
    sel = vsa.SelectParams(w.k_min, w.cum_mass, w.fixed_k or max(1, n_k // 5), w.n_anchor, w.anchor_rot)
    vsa.select_blocks(qp, kp, shape, w.bq, w.bk, w.scale, sel, counts, idx)
    return shape, q64, k16, counts, idx


CASES = [
    # (workload, heads, mode, topk, percentile, head flags)
    ("tiny", 2, 1, 4, 0.0, None),
    ("wan13b", 3, 2, 0, 0.99, [0, 1, 1]),
    ("wan13b", 2, 1, 8, 0.0, [1, 0]),
]


@pytest.mark.parametrize("case", CASES, ids=["tiny-top4", "wan13b-p99", "wan13b-top8"])
def test_noalloc_matches_workspace_entry_point_twice(case):
    name, H, mode, topk, pct, heads = case
    w = WORKLOADS[name]
    shape, q64, k16, counts, idx = _pooled_and_lists(w, H)
    n_r, n_t = w.n_pad // 64, w.n_pad // 16
    cap = n_t
    ws_bytes = vsa.select_micro_workspace_bytes(shape, mode, topk, pct, heads, cap)
    assert 0 < ws_bytes <= vsa.MICRO_NOALLOC_MAX_BYTES
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    ref_c = torch.empty(w.B, H, n_r, dtype=torch.int32, device="cuda")
    ref_i = torch.full((w.B, H, n_r, cap), -1, dtype=torch.int32, device="cuda")
    vsa.select_micro(q64, k16, counts, idx, shape, w.bq, w.bk, w.scale, mode, topk, pct, heads, cap, ref_c, ref_i, ws)
    assert vsa.read_device_status() == 0
    rc, ri = ref_c.cpu().numpy(), ref_i.cpu().numpy()
    assert rc.sum() > 0
    for call in range(2):
        got_c = torch.full((w.B, H, n_r), -5, dtype=torch.int32, device="cuda")
        got_i = torch.full((w.B, H, n_r, cap), -1, dtype=torch.int32, device="cuda")
        vsa.select_micro_noalloc(q64, k16, counts, idx, shape, w.bq, w.bk, w.scale, mode, topk, pct, heads, cap,
                                 got_c, got_i)
        assert vsa.read_device_status() == 0
        gc, gi = got_c.cpu().numpy(), got_i.cpu().numpy()
        assert np.array_equal(gc, rc), (name, call)
        for h in range(H):
            for r in range(n_r):
                c = rc[0, h, r]
                assert np.array_equal(gi[0, h, r, :c], ri[0, h, r, :c]), (name, call, h, r)


def test_noalloc_refuses_problems_beyond_its_fixed_scratch():
    w = WORKLOADS["hunyuan"]
    shape = vsa.Shape(1, 24, w.n_valid, w.n_pad, w.d)
    params, keep = vsa._micro_params(2, 0, 0.99, None, 16)
    assert vsa.select_micro_workspace_bytes(shape, 2, 0, 0.99, None, 16) > vsa.MICRO_NOALLOC_MAX_BYTES
    fake = ctypes.c_void_p(256)
    code = vsa.lib().vsa_select_micro_noalloc(fake, fake, fake, fake, ctypes.byref(shape), 128, 128, 0.088,
                                              ctypes.byref(params), fake, fake, None)
    del keep
    assert code == 7 and "scratch" in vsa.status_string(code)
