"""GPU parity of every step of the path against the fp64 CPU oracle.

All calls go through the C ABI (libvsa.so via the ctypes binding).  Inputs
are the seeded workloads of video_inputs; lists fed to the attention kernel in
the isolated attention tests come from the oracle, never the other way round.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
import oracle as orc
from video_inputs import WORKLOADS, make_qkv, micro_heads, round_to_bf16, sweep_points

from gpu_helpers import (GAP, LSE_TOL, O_TOL, assert_close_rows, compare_selection, oracle_select_per_head,
                         sample_blocks, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    torch.cuda.init()
    yield
    assert vsa.read_device_status() == 0


_CACHE = {}


def inputs(name, heads=None):
    key = (name, heads)
    if key not in _CACHE:
        w = WORKLOADS[name]
        _CACHE[key] = make_qkv(w, heads=heads)
    return _CACHE[key]


def shape_for(w, H=None):
    return vsa.Shape(w.B, w.H if H is None else H, w.n_valid, w.n_pad, w.d)


def lists_to_dev(kept, n_k, B, H, n_q):
    counts = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.zeros((B, H, n_q, n_k), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                row = np.asarray(kept[b][h][i], dtype=np.int32)
                counts[b, h, i] = row.size
                idx[b, h, i, :row.size] = row
    return torch.from_numpy(counts).cuda(), torch.from_numpy(idx).cuda()


# ---------------------------------------------------------------------------
# a1 pooling
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,heads", [("tiny", None), ("wan13b", (0, 3)), ("hunyuan", (0, 2))])
def test_pool_matches_oracle(name, heads):
    w = WORKLOADS[name]
    q, k, _ = inputs(name, heads)
    H = q.shape[1]
    shape = shape_for(w, H)
    dq, dk = to_dev(q), to_dev(k)
    f = lambda n: torch.empty(w.B, H, w.n_pad // n, w.d, device="cuda", dtype=torch.float32)
    qp, kp, q64, k16 = f(w.bq), f(w.bk), f(64), f(16)
    vsa.pool_qk(dq, dk, shape, w.bq, w.bk, qp, kp, q64, k16)
    torch.cuda.synchronize()
    for got, x, blk in ((qp, q, w.bq), (kp, k, w.bk), (q64, q, 64), (k16, k, 16)):
        want = orc.pool_block_means(x, blk, w.n_valid)
        err = np.abs(got.cpu().numpy().astype(np.float64) - want).max()
        assert err < 2e-5, (name, blk, err)


# ---------------------------------------------------------------------------
# a2 + a3 selection
# ---------------------------------------------------------------------------

def _gpu_select(w, q, k, with_mask=False):
    H = q.shape[1]
    shape = shape_for(w, H)
    dq, dk = to_dev(q), to_dev(k)
    n_q, n_k = w.n_pad // w.bq, w.n_pad // w.bk
    qp = torch.empty(w.B, H, n_q, w.d, device="cuda")
    kp = torch.empty(w.B, H, n_k, w.d, device="cuda")
    vsa.pool_qk(dq, dk, shape, w.bq, w.bk, qp, kp)
    counts = torch.empty(w.B, H, n_q, dtype=torch.int32, device="cuda")
    idx = torch.full((w.B, H, n_q, n_k), -7, dtype=torch.int32, device="cuda")
    mask = torch.empty(w.B, H, n_q, n_k, dtype=torch.uint8, device="cuda") if with_mask else None
    vsa.select_blocks(qp, kp, shape, w.bq, w.bk, w.scale,
                      vsa.SelectParams(w.k_min, w.cum_mass, w.fixed_k, w.n_anchor, w.anchor_rot), counts, idx, mask)
    torch.cuda.synchronize()
    return counts.cpu().numpy(), idx.cpu().numpy(), (mask.cpu().numpy() if with_mask else None)


@pytest.mark.parametrize("name,heads", [("tiny", None), ("wan13b", None), ("wan14b", (0, 4)), ("hunyuan", (0, 4))])
def test_select_blocks_bit_exact(name, heads):
    w = WORKLOADS[name]
    q, k, _ = inputs(name, heads)
    counts, idx, mask = _gpu_select(w, q, k, with_mask=True)
    kept, info, logw, probs, _, _ = oracle_select_per_head(q, k, w)
    n_exact, n_near, n_1e3 = compare_selection(counts, idx, kept, info, logw, probs, w, gpu_mask=mask)
    print(f"\n{name}: rows bit-exact {n_exact}, near-tie rows validity-checked {n_near}, gap<1e-3 rows {n_1e3}")
    assert n_exact >= 0.8 * (n_exact + n_near)


@pytest.mark.parametrize("point", [0, 4, 5, 9])
def test_select_sweep_points(point):
    frac, w = sweep_points()[point]
    q, k, _ = inputs("hunyuan", (0, 2))
    counts, idx, _ = _gpu_select(w, q, k)
    kept, info, logw, probs, _, _ = oracle_select_per_head(q, k, w)
    n_exact, n_near, _ = compare_selection(counts, idx, kept, info, logw, probs, w)
    assert n_exact >= 0.8 * (n_exact + n_near)
    n_q_valid = (w.n_valid + w.bq - 1) // w.bq
    assert np.all(counts[:, :, :n_q_valid] == min(w.fixed_k, w.n_k))
    assert np.all(counts[:, :, n_q_valid:] == 0)            # query blocks without a valid row keep nothing


def test_mask_to_lists_bit_exact():
    rng = np.random.default_rng(5)
    B, H, n = 1, 3, 700                       # 64-row blocks, n_pad = 44,800
    m = (rng.random((B, H, n, n)) < 0.3).astype(np.uint8)
    m[0, 0, 0] = 0
    m[0, 1, 1] = 1
    m[0, 2, 2] = 7                            # any nonzero byte means kept
    shape = vsa.Shape(B, H, n * 64, n * 64, 128)
    counts = torch.empty(B, H, n, dtype=torch.int32, device="cuda")
    idx = torch.empty(B, H, n, n, dtype=torch.int32, device="cuda")
    vsa.mask_to_lists(torch.from_numpy(m).cuda(), shape, 64, 64, counts, idx)
    c, ix = counts.cpu().numpy(), idx.cpu().numpy()
    for h in range(H):
        for i in range(n):
            want = np.nonzero(m[0, h, i])[0]
            assert c[0, h, i] == want.size and np.array_equal(ix[0, h, i, :want.size], want)


# ---------------------------------------------------------------------------
# a4 attention over given lists (oracle lists -> GPU)
# ---------------------------------------------------------------------------

def _attention_case(w, q, k, v, kept, blocks, o_fp32=False):
    B, H = q.shape[0], q.shape[1]
    n_q, n_k = w.n_pad // w.bq, w.n_pad // w.bk
    counts, idx = lists_to_dev(kept, n_k, B, H, n_q)
    shape = vsa.Shape(B, H, w.n_valid, w.n_pad, w.d)
    o = torch.empty(B, H, w.n_pad, w.d, device="cuda", dtype=torch.float32 if o_fp32 else torch.bfloat16)
    lse = torch.empty(B, H, w.n_pad, device="cuda")
    vsa.block_sparse_fwd(to_dev(q), to_dev(k), to_dev(v), shape, w.bq, w.bk, counts, idx, n_k, w.scale, o, lse)
    assert vsa.read_device_status() == 0
    Og = o.float().cpu().numpy()
    Lg = lse.cpu().numpy()
    O, L = orc.block_sparse_attention(q, k, v, kept, w.bq, w.bk, w.n_valid, w.scale, rows=blocks)
    rows = [(b, h, i * w.bq, (i + 1) * w.bq) for b, h, i in blocks]
    return assert_close_rows(Og, Lg, O, L, rows, bf16_out=not o_fp32)


def test_attention_tiny_all_rows():
    w = WORKLOADS["tiny"]
    q, k, v = inputs("tiny")
    kept, *_ = oracle_select_per_head(q, k, w)
    blocks = [(0, h, i) for h in range(w.H) for i in range(w.n_q)]
    print("\ntiny attention worst |dO|, |dLSE|:", _attention_case(w, q, k, v, kept, blocks))


def test_attention_dense_equals_full_attention():
    w = WORKLOADS["wan13b"]
    q, k, v = inputs("wan13b", (0, 1))
    n_q, n_k = w.n_pad // w.bq, w.n_pad // w.bk
    kept = [[[np.arange(n_k) for _ in range(n_q)]]]
    blocks = [(0, 0, 0), (0, 0, 100), (0, 0, n_q - 1)]
    print("\ndense worst:", _attention_case(w, q, k, v, kept, blocks, o_fp32=True))


@pytest.mark.parametrize("name", ["wan13b", "wan14b", "hunyuan"])
def test_attention_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = inputs(name, (0, 2))
    kept, *_ = oracle_select_per_head(q, k, w)
    blocks = sample_blocks(w, 6, seed=1, heads=2)
    print(f"\n{name} attention worst fp32 O:", _attention_case(w, q, k, v, kept, blocks, o_fp32=True))
    print(f"{name} attention worst bf16 O (beyond rounding):", _attention_case(w, q, k, v, kept, blocks))


@pytest.mark.parametrize("point", [1, 6, 9])
def test_attention_sweep_points(point):
    frac, w = sweep_points()[point]
    q, k, v = inputs("hunyuan", (0, 1))
    kept, *_ = oracle_select_per_head(q, k, w)
    blocks = sample_blocks(w, 4, seed=2, heads=1)
    print(f"\nsweep {w.name} worst:", _attention_case(w, q, k, v, kept, blocks))


@pytest.mark.parametrize("n_pad,list_rows,seg", [(512, 128, 32), (512, 64, 32), (512, 64, 128), (512, 128, 16),
                                                 (512, 128, 128), (384, 128, 128), (640, 128, 128),
                                                 (384, 64, 128), (640, 64, 128)])
def test_attention_ragged_and_empty_rows(n_pad, list_rows, seg):
    """n_valid not a multiple of the block, a row with an empty list, lists of
    different lengths in one 128-row tile (64-row lists), short segments, and
    the two-tile path (128-row lists, and 64-row lists of 128-key blocks, where
    each half of a tile keeps its own blocks) with an even and an odd number
    of query tiles."""
    rng = np.random.default_rng(9 + n_pad + seg)
    B, H, d = 1, 2, 128
    n_valid = n_pad - 75
    q, k, v = (round_to_bf16(rng.standard_normal((B, H, n_pad, d)).astype(np.float32)) for _ in range(3))
    for x in (q, k, v):
        x[:, :, n_valid:] = 0
    n_l, n_s = n_pad // list_rows, n_pad // seg
    kept = [[[np.sort(rng.choice(n_s, size=int(rng.integers(0, n_s // 2 + 1)), replace=False))
              for _ in range(n_l)] for _ in range(H)]]
    kept[0][0][1] = np.zeros(0, dtype=np.int64)
    kept[0][1][0] = np.arange(n_s)                      # one dense row
    counts, idx = lists_to_dev(kept, n_s, B, H, n_l)
    shape = vsa.Shape(B, H, n_valid, n_pad, d)
    o = torch.empty(B, H, n_pad, d, device="cuda")
    lse = torch.empty(B, H, n_pad, device="cuda")
    scale = 1 / math.sqrt(d)
    vsa.block_sparse_fwd(to_dev(q), to_dev(k), to_dev(v), shape, list_rows, seg, counts, idx, n_s, scale, o, lse)
    assert vsa.read_device_status() == 0
    mask = orc.token_mask(kept, None, n_pad, list_rows, seg, n_valid)
    O, L = orc.masked_attention_bruteforce(q, k, v, mask, scale)
    assert_close_rows(o.cpu().numpy(), lse.cpu().numpy(), O, L, [(0, h, 0, n_pad) for h in range(H)])


@pytest.mark.parametrize("list_rows,seg", [(128, 128), (64, 128), (64, 16)])
def test_attention_head_subset(list_rows, seg):
    """vsa_block_sparse_fwd_heads on some (batch, head) pairs, given in any
    order, writes for them exactly what the all-heads call writes, leaves the
    other heads' rows untouched, and an out-of-range entry latches BAD_INDEX
    without disturbing the valid entries."""
    rng = np.random.default_rng(21 + seg)
    B, H, n_pad, d = 2, 3, 640, 128
    n_valid = n_pad - 40
    q, k, v = (to_dev(round_to_bf16(rng.standard_normal((B, H, n_pad, d)).astype(np.float32))) for _ in range(3))
    n_l, n_s = n_pad // list_rows, n_pad // seg
    kept = [[[np.sort(rng.choice(n_s, size=int(rng.integers(1, n_s // 2 + 1)), replace=False))
              for _ in range(n_l)] for _ in range(H)] for _ in range(B)]
    counts, idx = lists_to_dev(kept, n_s, B, H, n_l)
    shape = vsa.Shape(B, H, n_valid, n_pad, d)
    scale = 1 / math.sqrt(d)
    o_all = torch.empty(B * H, n_pad, d, device="cuda")
    l_all = torch.empty(B * H, n_pad, device="cuda")
    vsa.block_sparse_fwd(q, k, v, shape, list_rows, seg, counts, idx, n_s, scale, o_all, l_all)
    for sub, status in (([4, 0, 3], 0), ([5, B * H + 7, 1], 5)):
        o = torch.full((B * H, n_pad, d), 7.0, device="cuda")
        lse = torch.full((B * H, n_pad), 5.0, device="cuda")
        heads = torch.tensor(sub, dtype=torch.int32, device="cuda")
        vsa.block_sparse_fwd(q, k, v, shape, list_rows, seg, counts, idx, n_s, scale, o, lse, heads=heads)
        assert vsa.read_device_status() == status
        for bh in range(B * H):
            if bh in sub:
                assert torch.equal(o[bh], o_all[bh]) and torch.equal(lse[bh], l_all[bh]), (sub, bh)
            else:
                assert torch.all(o[bh] == 7.0) and torch.all(lse[bh] == 5.0), (sub, bh)


def test_attention_long_lists_both_union_paths():
    """64-row lists of 16-key segments as long as the sequence allows: tiles
    whose two lists fit the shared-memory staging (up to 2048 entries each,
    union up to 4096) take the staged union; a tile with a longer list is
    merged from global memory.  Rows of both kinds, and a short neighbour,
    are compared with the oracle."""
    rng = np.random.default_rng(77)
    B, H, d, seg, list_rows = 1, 1, 128, 16, 64
    n_pad = seg * 2304
    n_valid = n_pad - 9
    q, k, v = (round_to_bf16(rng.standard_normal((B, H, n_pad, d)).astype(np.float32)) for _ in range(3))
    n_l, n_s = n_pad // list_rows, n_pad // seg
    pick = lambda n: np.sort(rng.choice(n_s, size=n, replace=False))
    kept = [[[pick(int(rng.integers(0, 40))) for _ in range(n_l)]]]
    sizes = {2: 2100, 3: 50,            # tile 1: one list past the staging size (global merge)
             10: 2048, 11: 2048,        # tile 5: both at the staging size (staged union)
             20: 2300, 21: 2200,        # tile 10: both long
             n_l - 2: 1500, n_l - 1: 2048}
    for r, n in sizes.items():
        kept[0][0][r] = pick(n)
    counts, idx = lists_to_dev(kept, n_s, B, H, n_l)
    shape = vsa.Shape(B, H, n_valid, n_pad, d)
    o = torch.empty(B, H, n_pad, d, device="cuda")
    lse = torch.empty(B, H, n_pad, device="cuda")
    scale = 1 / math.sqrt(d)
    vsa.block_sparse_fwd(to_dev(q), to_dev(k), to_dev(v), shape, list_rows, seg, counts, idx, n_s, scale, o, lse)
    assert vsa.read_device_status() == 0
    rows = [(0, 0, r) for r in sorted(set(sizes) | {0, 1, 30})]
    O, L = orc.block_sparse_attention(q, k, v, kept, list_rows, seg, n_valid, scale, rows=rows)
    assert_close_rows(o.cpu().numpy(), lse.cpu().numpy(), O, L,
                      [(b, h, r * list_rows, (r + 1) * list_rows) for b, h, r in rows])


def test_attention_64row_lists_on_both_kernels():
    """64-row lists of 128-key blocks: up to 1024 key blocks they run on the
    two-tile kernel (each tile walks the union of its halves' lists), beyond
    that on the single-tile kernel.  A layer of 1032 key blocks, with rows
    where one half of a tile keeps nothing, rows where both halves keep the
    same blocks and rows with disjoint lists, against the oracle on sampled
    rows; the same lists on the first 1024 blocks take the two-tile kernel."""
    rng = np.random.default_rng(5)
    B, H, d, seg, list_rows = 1, 1, 64, 128, 64
    for n_blocks in (1032, 1024):
        n_pad = seg * n_blocks
        n_valid = n_pad - 33
        q, k, v = (round_to_bf16(rng.standard_normal((B, H, n_pad, d)).astype(np.float32)) for _ in range(3))
        n_l, n_s = n_pad // list_rows, n_pad // seg
        pick = lambda n: np.sort(rng.choice(n_s, size=n, replace=False))
        kept = [[[pick(int(rng.integers(1, 12))) for _ in range(n_l)]]]
        kept[0][0][4] = np.zeros(0, dtype=np.int64)          # tile 2: half 0 keeps nothing
        kept[0][0][7] = kept[0][0][6].copy()                  # tile 3: both halves alike
        kept[0][0][n_l - 1] = np.array([n_s - 1])             # last tile: the ragged block only
        counts, idx = lists_to_dev(kept, n_s, B, H, n_l)
        shape = vsa.Shape(B, H, n_valid, n_pad, d)
        o = torch.empty(B, H, n_pad, d, device="cuda")
        lse = torch.empty(B, H, n_pad, device="cuda")
        scale = 1 / math.sqrt(d)
        vsa.block_sparse_fwd(to_dev(q), to_dev(k), to_dev(v), shape, list_rows, seg, counts, idx, n_s, scale, o,
                             lse)
        assert vsa.read_device_status() == 0
        rows = [(0, 0, r) for r in (0, 1, 4, 5, 6, 7, 501, n_l - 2, n_l - 1)]
        O, L = orc.block_sparse_attention(q, k, v, kept, list_rows, seg, n_valid, scale, rows=rows)
        assert_close_rows(o.cpu().numpy(), lse.cpu().numpy(), O, L,
                          [(b, h, r * list_rows, (r + 1) * list_rows) for b, h, r in rows])


def test_attention_two_tile_kernel_long_lists_from_global_memory():
    """128-row lists of 128-key blocks longer than the 1024 entries the
    two-tile kernel stages in shared memory: such a pair of tiles walks the
    union of its lists from global memory instead.  A layer of 1032 key
    blocks: one tile keeping 1030 blocks next to a tile keeping a few, a pair
    of long lists, and short pairs, against the oracle on sampled rows."""
    rng = np.random.default_rng(21)
    B, H, d, seg, list_rows = 1, 1, 64, 128, 128
    n_blocks = 1032
    n_pad = seg * n_blocks
    n_valid = n_pad - 70
    q, k, v = (round_to_bf16(rng.standard_normal((B, H, n_pad, d)).astype(np.float32)) for _ in range(3))
    n_l = n_s = n_blocks
    pick = lambda n: np.sort(rng.choice(n_s, size=n, replace=False))
    kept = [[[pick(int(rng.integers(1, 9))) for _ in range(n_l)]]]
    sizes = {2: 1030, 3: 5,            # pair 1: one list past the staging size
             10: 1025, 11: 1032,       # pair 5: both long, one of them dense
             n_l - 1: 1031}            # last pair: the ragged block among them
    for r, n in sizes.items():
        kept[0][0][r] = pick(n)
    counts, idx = lists_to_dev(kept, n_s, B, H, n_l)
    shape = vsa.Shape(B, H, n_valid, n_pad, d)
    o = torch.empty(B, H, n_pad, d, device="cuda")
    lse = torch.empty(B, H, n_pad, device="cuda")
    scale = 1 / math.sqrt(d)
    vsa.block_sparse_fwd(to_dev(q), to_dev(k), to_dev(v), shape, list_rows, seg, counts, idx, n_s, scale, o, lse)
    assert vsa.read_device_status() == 0
    rows = [(0, 0, r) for r in (0, 1, 2, 3, 10, 11, 400, n_l - 2, n_l - 1)]
    O, L = orc.block_sparse_attention(q, k, v, kept, list_rows, seg, n_valid, scale, rows=rows)
    assert_close_rows(o.cpu().numpy(), lse.cpu().numpy(), O, L,
                      [(b, h, r * list_rows, (r + 1) * list_rows) for b, h, r in rows])


def test_attention_bad_64row_list_latches_status():
    """A descending 64-row list in the two-tile kernel: the status word reads
    VSA_ERR_BAD_INDEX and the CTA's tiles write O = 0, LSE = -inf."""
    B, H, n_pad, d = 1, 1, 256, 128
    q = torch.zeros(B, H, n_pad, d, device="cuda", dtype=torch.bfloat16)
    counts = torch.tensor([[[1, 2, 1, 0]]], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[[[0, 0], [1, 0], [1, 0], [0, 0]]]], dtype=torch.int32, device="cuda")   # row 1 descending
    o = torch.empty(B, H, n_pad, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, H, n_pad, device="cuda")
    vsa.block_sparse_fwd(q, q, q, vsa.Shape(B, H, n_pad, n_pad, d), 64, 128, counts, idx, 2, 0.1, o, lse)
    assert vsa.read_device_status() == 5
    assert torch.all(o == 0) and torch.all(torch.isinf(lse))
    assert vsa.read_device_status() == 0


def test_attention_bad_list_latches_status():
    B, H, n_pad, d = 1, 1, 256, 128
    q = torch.zeros(B, H, n_pad, d, device="cuda", dtype=torch.bfloat16)
    counts = torch.tensor([[[2, 1]]], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[[[1, 0], [5, 0]]]], dtype=torch.int32, device="cuda")   # descending; out of range
    o = torch.empty(B, H, n_pad, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, H, n_pad, device="cuda")
    vsa.block_sparse_fwd(q, q, q, vsa.Shape(B, H, n_pad, n_pad, d), 128, 128, counts, idx, 2, 0.1, o, lse)
    assert vsa.read_device_status() == 5
    assert torch.all(o == 0) and torch.all(torch.isinf(lse))
    assert vsa.read_device_status() == 0                      # reading clears it


def test_bounded_wait_times_out_and_device_stays_usable():
    """Failure detection without a fault: a wait that nothing completes gives
    up after its limit, the status reads VSA_ERR_TIMEOUT, reading clears it,
    and the next attention call runs normally."""
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    vsa.selftest_wait_timeout(50_000_000)          # 50 ms
    t1.record()
    assert vsa.read_device_status() == 6
    assert t0.elapsed_time(t1) >= 45.0
    assert vsa.read_device_status() == 0
    test_attention_tiny_all_rows()
    assert vsa.read_device_status() == 0


def test_softmax_exp2_matches_cuda_exp2_within_its_bound():
    """The exponential the Macro softmax runs on the FMA pipe for part of its
    logits, against CUDA's exp2 (torch.exp2 on the device): relative error
    within the polynomial's 7.5e-5 plus fp32 evaluation rounding over the
    logit range the softmax produces ([-125, 8] after the lazy-rescale
    threshold of 2^8), every integer and half-integer included; masked
    logits (-inf) and anything below -125 give 2^-125 x (1 +- 7.5e-5)."""
    g = torch.Generator(device="cuda").manual_seed(11)
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20, device="cuda"),
                   torch.arange(-125.0, 8.5, 0.5, device="cuda"),
                   torch.rand(100_001, device="cuda", generator=g) * 133.0 - 125.0])
    y = torch.empty_like(x)
    vsa.selftest_exp2(x, y)
    ref = torch.exp2(x)
    rel = ((y.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel <= 7.5e-5 + 4 * 2.0 ** -24, rel
    low = torch.tensor([-float("inf"), -1000.0, -126.5, -125.0], device="cuda")
    y_low = torch.empty_like(low)
    vsa.selftest_exp2(low, y_low)
    assert torch.all(y_low == y_low[-1])
    assert abs(y_low[-1].item() / 2.0 ** -125 - 1.0) <= 7.5e-5
    # odd length: the last element of the final pair
    xo = torch.tensor([0.0, 1.0, -2.0], device="cuda")
    yo = torch.full_like(xo, float("nan"))
    vsa.selftest_exp2(xo, yo)
    assert torch.allclose(yo, torch.exp2(xo), rtol=8e-5, atol=0.0)


# ---------------------------------------------------------------------------
# a6 merge
# ---------------------------------------------------------------------------

def test_lse_merge_kernel():
    rng = np.random.default_rng(3)
    B, H, n_pad, d = 1, 2, 256, 64
    oa, ob = rng.normal(size=(2, B, H, n_pad, d)).astype(np.float32)
    la, lb = rng.normal(scale=3, size=(2, B, H, n_pad)).astype(np.float32)
    la[0, 0, :10] = -np.inf
    lb[0, 0, 5:15] = -np.inf
    O, L = orc.lse_merge(oa, la, ob, lb)
    t = lambda x: torch.from_numpy(x).cuda()
    for out_dtype, tol in ((torch.float32, 1e-5), (torch.bfloat16, 1e-2)):
        o = torch.empty(B, H, n_pad, d, device="cuda", dtype=out_dtype)
        lo = torch.empty(B, H, n_pad, device="cuda")
        vsa.lse_merge(t(oa), t(la), t(ob), t(lb), vsa.Shape(B, H, n_pad, n_pad, d), o, lo)
        Lg = lo.cpu().numpy()
        assert np.abs(o.float().cpu().numpy() - O).max() < tol
        fin = np.isfinite(L)
        assert np.array_equal(np.isfinite(Lg), fin)
        assert np.abs(Lg[fin] - L[fin]).max() < 1e-5


# ---------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("micro_mode", [1, 2])
def test_path_two_batches_every_row(micro_mode):
    """B = 2 through the whole path: batch-major (batch, head) indexing in
    every kernel, Micro head flags repeated per batch element, the per-head
    percentile taken per (batch, head) slot, and the Micro pass and its fp32
    Macro output restricted to the flagged heads of both batch elements."""
    import dataclasses
    w = dataclasses.replace(WORKLOADS["tiny"], B=2, micro_mode=micro_mode, micro_percentile=0.9, fixed_k=2)
    q, k, v = make_qkv(w)
    assert q.shape[0] == 2 and not np.array_equal(q[0], q[1])
    heads = np.array([1, 0], dtype=np.uint8) if micro_mode == 2 else micro_heads(w)
    res = orc.forward(q, k, v, w, head_enable=heads)
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    out = run(to_dev(q), to_dev(k), to_dev(v))
    assert vsa.read_device_status() == 0
    counts, idx = out["counts"].cpu().numpy(), out["idx"].cpu().numpy()
    mc, mi = out["m_counts"].cpu().numpy(), out["m_idx"].cpu().numpy()
    for b in range(2):
        for h in range(w.H):
            for i in range(w.n_q):
                assert np.array_equal(idx[b, h, i, :counts[b, h, i]], res["kept"][b][h][i]), (b, h, i)
            for r in range(w.n_pad // 64):
                assert np.array_equal(mi[b, h, r, :mc[b, h, r]], res["tiles"][b][h][r]), (b, h, r)
    assert_close_rows(out["o"].float().cpu().numpy(), out["lse"].cpu().numpy(), res["O"], res["LSE"],
                      [(b, h, 0, w.n_pad) for b in range(2) for h in range(w.H)], bf16_out=True)


def test_path_tiny_every_row():
    w = WORKLOADS["tiny"]
    q, k, v = inputs("tiny")
    heads = micro_heads(w)
    res = orc.forward(q, k, v, w, head_enable=heads)
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    out = run(to_dev(q), to_dev(k), to_dev(v))
    assert vsa.read_device_status() == 0
    counts = out["counts"].cpu().numpy()
    idx = out["idx"].cpu().numpy()
    for h in range(w.H):
        for i in range(w.n_q):
            assert np.array_equal(idx[0, h, i, :counts[0, h, i]], res["kept"][0][h][i])
    mc = out["m_counts"].cpu().numpy()
    mi = out["m_idx"].cpu().numpy()
    for h in range(w.H):
        for r in range(w.n_pad // 64):
            assert np.array_equal(mi[0, h, r, :mc[0, h, r]], res["tiles"][0][h][r]), (h, r)
    worst = assert_close_rows(out["o"].float().cpu().numpy(), out["lse"].cpu().numpy(), res["O"], res["LSE"],
                              [(0, h, 0, w.n_pad) for h in range(w.H)], bf16_out=True)
    print("\ntiny path worst:", worst)


def test_path_hunyuan_sampled():
    """The benchmark's launch configuration: the whole hunyuan path (Macro
    fixed 20%, Micro percentile in 6 of 24 heads) on all heads; sampled rows
    compared with the oracle."""
    w = WORKLOADS["hunyuan"]
    q, k, v = inputs("hunyuan")
    heads = micro_heads(w)
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    out = run(to_dev(q), to_dev(k), to_dev(v))
    assert vsa.read_device_status() == 0
    counts = out["counts"].cpu().numpy()
    idx = out["idx"].cpu().numpy()
    mc = out["m_counts"].cpu().numpy()
    mi = out["m_idx"].cpu().numpy()
    Og = out["o"].float().cpu().numpy()
    Lg = out["lse"].cpu().numpy()
    kept, info, logw, probs, _, _ = oracle_select_per_head(q, k, w)
    n_exact, n_near, _ = compare_selection(counts, idx, kept, info, logw, probs, w)
    assert n_exact >= 0.8 * (n_exact + n_near)
    # Micro selection per enabled head, tiles decided away from tau compared exactly
    q64 = np.zeros((1, w.H, w.n_pad // 64, w.d))
    k16 = np.zeros((1, w.H, w.n_pad // 16, w.d))
    for h in np.nonzero(heads)[0]:
        q64[0, h] = orc.pool_block_means(q[:, h:h + 1], 64, w.n_valid)[0, 0]
        k16[0, h] = orc.pool_block_means(k[:, h:h + 1], 16, w.n_valid)[0, 0]
    tiles, minfo = orc.select_micro_percentile(q64, k16, kept, w.bq, w.bk, w.n_valid, w.scale,
                                               w.micro_percentile, heads, with_info=True)
    for h in range(w.H):
        if not heads[h]:
            assert np.all(mc[0, h] == 0)
            continue
        inf = minfo[0][h]
        far = inf["cand"] & (np.abs(inf["S"] - inf["tau"]) >= GAP)
        sel_o = np.zeros_like(far)
        for r, t in enumerate(tiles[0][h]):
            sel_o[r, t] = True
        sel_g = np.zeros_like(far)
        for r in range(far.shape[0]):
            sel_g[r, mi[0, h, r, :mc[0, h, r]]] = True
        assert np.array_equal(sel_g[far], sel_o[far]), h
        assert not np.any(sel_g & ~inf["cand"])
        assert abs(int(sel_g.sum()) - int(sel_o.sum())) <= int((inf["cand"] & ~far).sum())
    # output rows: blocks whose Macro row and both Micro rows match the oracle exactly
    blocks = sample_blocks(w, 8, seed=4)
    rows = []
    for b, h, i in blocks:
        if not np.array_equal(idx[b, h, i, :counts[b, h, i]], kept[b][h][i]):
            continue
        ok = all(np.array_equal(mi[b, h, r, :mc[b, h, r]], tiles[b][h][r]) for r in (2 * i, 2 * i + 1))
        if ok:
            rows.append((b, h, i))
    assert len(rows) >= 4
    O_M, L_M = orc.block_sparse_attention(q, k, v, kept, w.bq, w.bk, w.n_valid, w.scale, rows=rows)
    mrows = [(b, h, r) for b, h, i in rows for r in (2 * i, 2 * i + 1)]
    O_u, L_u = orc.micro_attention(q, k, v, tiles, w.n_valid, w.scale, rows=mrows)
    O, L = orc.lse_merge(O_M, L_M, O_u, L_u)
    worst = assert_close_rows(Og, Lg, O, L, [(b, h, i * 128, i * 128 + 128) for b, h, i in rows], bf16_out=True)
    print("\nhunyuan path worst:", worst, "rows", rows)


@pytest.mark.parametrize("name,heads,chunk", [("tiny", None, 1), ("hunyuan", (0, 3), 2)])
def test_forward_host_matches_device_path(name, heads, chunk):
    """The host-buffer API (chunks of heads pipelined over copy and compute
    streams) returns exactly what the device path returns for all heads."""
    w = WORKLOADS[name]
    q, k, v = inputs(name, heads)
    H = q.shape[1]
    flags = micro_heads(w)[:H] if w.micro_mode else None
    if flags is not None and w.micro_mode == 2:
        flags = np.array([1] + [0] * (H - 1), dtype=np.uint8)   # at least one Micro head in the cut
    cfg = vsa.PathConfig.from_workload(w, flags)
    ref = vsa.SparseVideoAttention(cfg)(to_dev(q), to_dev(k), to_dev(v))
    o_ref, l_ref = ref["o"].cpu(), ref["lse"].cpu()
    pin = lambda x: torch.from_numpy(x).to(torch.bfloat16).pin_memory()
    ho = torch.empty(o_ref.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(l_ref.shape, dtype=torch.float32).pin_memory()
    run = vsa.SparseVideoAttention(cfg)
    run.forward_host(pin(q), pin(k), pin(v), ho, hl, chunk_heads=chunk)
    assert vsa.read_device_status() == 0
    assert torch.equal(ho, o_ref)
    assert torch.equal(torch.isinf(hl), torch.isinf(l_ref))
    fin = torch.isfinite(l_ref)
    assert torch.equal(hl[fin], l_ref[fin])


def test_status_words_bound_to_streams_keep_callers_apart():
    """Two callers on two streams, each with its own status word in its own
    memory: a bad list on one stream latches BAD_INDEX in that caller's word
    only, a wait that times out on it aborts nothing on the other, and
    unbinding returns the stream to the process-wide word."""
    B, H, n_pad, d = 1, 1, 256, 128
    q = torch.zeros(B, H, n_pad, d, device="cuda", dtype=torch.bfloat16)
    bad_counts = torch.tensor([[[2, 1]]], dtype=torch.int32, device="cuda")
    bad_idx = torch.tensor([[[[1, 0], [5, 0]]]], dtype=torch.int32, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    w1 = torch.full((2,), 77, dtype=torch.int32, device="cuda")
    w2 = torch.full((2,), 77, dtype=torch.int32, device="cuda")
    vsa.bind_status_word(w1, s1)
    vsa.bind_status_word(w2, s2)
    try:
        o1 = torch.empty(B, H, n_pad, d, device="cuda", dtype=torch.bfloat16)
        l1 = torch.empty(B, H, n_pad, device="cuda")
        with torch.cuda.stream(s1):
            vsa.block_sparse_fwd(q, q, q, vsa.Shape(B, H, n_pad, n_pad, d), 128, 128, bad_counts, bad_idx, 2, 0.1,
                                 o1, l1, stream=s1)
            vsa.selftest_wait_timeout(20_000_000, stream=s1)      # 20 ms
        with torch.cuda.stream(s2):
            test_attention_tiny_all_rows()
        s1.synchronize()
        s2.synchronize()
        assert int(w1[0]) == 5 and int(w1[1]) == 1        # first error kept; the timeout raised its flag
        assert int(w2[0]) == 0 and int(w2[1]) == 0
        assert vsa.read_device_status(s2) == 0
        assert vsa.read_device_status(s1) == 5
        assert int(w1[0]) == 0 and int(w1[1]) == 0        # reading cleared the caller's word
        assert vsa.read_device_status() == 0              # the process-wide word saw nothing
    finally:
        vsa.bind_status_word(None, s1)
        vsa.bind_status_word(None, s2)
    # unbound again: errors land in the process-wide word
    with torch.cuda.stream(s1):
        vsa.block_sparse_fwd(q, q, q, vsa.Shape(B, H, n_pad, n_pad, d), 128, 128, bad_counts, bad_idx, 2, 0.1, o1, l1,
                             stream=s1)
    assert vsa.read_device_status(s1) == 5
    assert int(w1[0]) == 0
