"""Memory-safety and determinism checks of the whole path, in place of a
sanitizer (compute-sanitizer is closed on this machine):

  * canaries: every output of every stage (pooled means, kept lists, block
    mask, Macro and Micro outputs, Micro lists) lives inside a larger device
    buffer whose guard regions before and after it hold a byte pattern; after
    each call the guards must be intact (an out-of-bounds write shows here);
  * poisoning: outputs start as NaN (floats) or as an out-of-range pattern
    (integers), and the Micro workspace as 0xFF bytes, so a read of a value
    that a kernel never wrote, or of scratch that a call should have cleared,
    changes the result; the results must equal, bit for bit, those of the same
    path run on freshly allocated buffers;
  * determinism: two runs of block selection, Micro selection and the whole
    path on the full HunyuanVideo-like layer give bit-identical lists and
    outputs.

All calls go through the C ABI.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
from video_inputs import WORKLOADS, make_qkv, micro_heads

from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu

PAD = 4096          # guard bytes on each side (keeps 256-byte alignment)
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    torch.cuda.init()
    yield
    assert vsa.read_device_status() == 0


class Guarded:
    """A device tensor of ``shape``/``dtype`` inside a buffer with guard bytes."""

    def __init__(self, shape, dtype, poison):
        n = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((PAD + n + PAD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[PAD:PAD + n].view(dtype).view(*shape)
        if poison == "nan":
            self.t.fill_(float("nan"))
        elif poison == "ff":
            self.raw[PAD:PAD + n].fill_(0xFF)
        else:
            self.t.fill_(poison)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.raw[:PAD] == CANARY).all()) and bool((self.raw[PAD + self.n:] == CANARY).all())


def _stepwise(w, dq, dk, dv, flags):
    """The path stage by stage on guarded, poisoned buffers; guards checked after
    every stage.  Returns the outputs as host arrays."""
    B, H, n_pad, d = dq.shape
    shape = vsa.Shape(B, H, w.n_valid, n_pad, d)
    n_q, n_k, n_r, n_t = n_pad // w.bq, n_pad // w.bk, n_pad // 64, n_pad // 16
    f32, i32 = torch.float32, torch.int32
    g = {
        "q_pool": Guarded((B, H, n_q, d), f32, "nan"), "k_pool": Guarded((B, H, n_k, d), f32, "nan"),
        "q64": Guarded((B, H, n_r, d), f32, "nan"), "k16": Guarded((B, H, n_t, d), f32, "nan"),
        "counts": Guarded((B, H, n_q), i32, -7), "idx": Guarded((B, H, n_q, n_k), i32, 0x7fffffff),
        "mask": Guarded((B, H, n_q, n_k), torch.uint8, 0xEE),
        "o": Guarded((B, H, n_pad, d), torch.bfloat16, "nan"), "lse": Guarded((B, H, n_pad), f32, "nan"),
    }
    vsa.pool_qk(dq, dk, shape, w.bq, w.bk, g["q_pool"].t, g["k_pool"].t, g["q64"].t, g["k16"].t)
    assert all(g[n].intact() for n in ("q_pool", "k_pool", "q64", "k16"))
    vsa.select_blocks(g["q_pool"].t, g["k_pool"].t, shape, w.bq, w.bk, w.scale,
                      vsa.SelectParams(w.k_min, w.cum_mass, w.fixed_k, w.n_anchor, w.anchor_rot),
                      g["counts"].t, g["idx"].t, g["mask"].t)
    assert all(g[n].intact() for n in ("counts", "idx", "mask"))
    micro = w.micro_mode != 0
    if not micro:
        vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, g["counts"].t, g["idx"].t, n_k, w.scale, g["o"].t,
                             g["lse"].t)
        assert g["o"].intact() and g["lse"].intact()
    else:
        cap = n_t
        g.update({
            "o_macro": Guarded((B, H, n_pad, d), f32, "nan"), "lse_macro": Guarded((B, H, n_pad), f32, "nan"),
            "m_counts": Guarded((B, H, n_r), i32, -7), "m_idx": Guarded((B, H, n_r, cap), i32, 0x7fffffff),
        })
        ws_bytes = vsa.select_micro_workspace_bytes(shape, w.micro_mode, w.micro_topk, w.micro_percentile,
                                                    list(flags), cap)
        g["ws"] = Guarded((ws_bytes,), torch.uint8, "ff")
        rep = [b * H + h for b in range(B) for h in range(H) if flags[h]]
        plain = [b * H + h for b in range(B) for h in range(H) if not flags[h]]
        as_dev = lambda x: torch.tensor(x, dtype=torch.int32, device="cuda")
        if plain:
            vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, g["counts"].t, g["idx"].t, n_k, w.scale, g["o"].t,
                                 g["lse"].t, heads=as_dev(plain))
        vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, g["counts"].t, g["idx"].t, n_k, w.scale,
                             g["o_macro"].t, g["lse_macro"].t, heads=as_dev(rep))
        assert all(g[n].intact() for n in ("o", "lse", "o_macro", "lse_macro"))
        vsa.select_micro(g["q64"].t, g["k16"].t, g["counts"].t, g["idx"].t, shape, w.bq, w.bk, w.scale,
                         w.micro_mode, w.micro_topk, w.micro_percentile, list(flags), cap, g["m_counts"].t,
                         g["m_idx"].t, g["ws"].t)
        assert all(g[n].intact() for n in ("m_counts", "m_idx", "ws"))
        vsa.block_sparse_fwd(dq, dk, dv, shape, 64, 16, g["m_counts"].t, g["m_idx"].t, cap, w.scale, g["o"].t,
                             g["lse"].t, g["o_macro"].t, g["lse_macro"].t, heads=as_dev(rep))
        assert all(g[n].intact() for n in ("o", "lse", "o_macro", "lse_macro", "m_counts", "m_idx"))
    assert vsa.read_device_status() == 0
    return {n: x.t.cpu() for n, x in g.items() if n != "ws"}


@pytest.mark.parametrize("name,heads,flags", [("tiny", None, None), ("wan13b", (0, 3), None),
                                              ("wan14b", (0, 2), None), ("hunyuan", (0, 4), (1, 0, 0, 1))])
def test_guards_intact_and_poison_free(name, heads, flags):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    if w.micro_mode:
        flags = np.array(flags if flags is not None else micro_heads(w)[:H], dtype=np.uint8)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    got = _stepwise(w, dq, dk, dv, flags)
    ref = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, flags))(dq, dk, dv)
    assert vsa.read_device_status() == 0
    counts = ref["counts"].cpu()
    assert torch.equal(got["counts"], counts)
    idx_g, idx_r = got["idx"], ref["idx"].cpu()
    for row in np.ndindex(*counts.shape):
        c = int(counts[row])
        assert torch.equal(idx_g[row][:c], idx_r[row][:c]), row
        assert torch.all(idx_g[row][c:] == 0x7fffffff), row          # slots past the count untouched
    mask = got["mask"].numpy()
    assert set(np.unique(mask).tolist()) <= {0, 1}
    assert torch.equal(got["o"].view(torch.int16), ref["o"].cpu().view(torch.int16))   # bit-identical, NaN-free
    assert torch.equal(got["lse"].view(torch.int32), ref["lse"].cpu().view(torch.int32))
    assert not torch.isnan(got["o"].float()).any() and not torch.isnan(got["lse"]).any()
    if w.micro_mode:
        mc = ref["m_counts"].cpu()
        assert torch.equal(got["m_counts"], mc)
        mi_r = ref["m_idx"].cpu()
        for row in np.ndindex(*mc.shape):
            c = int(mc[row])
            assert torch.equal(got["m_idx"][row][:c], mi_r[row][:c]), row


def test_two_runs_bit_identical_on_the_full_layer():
    """Selection (block and Micro) and the whole path, twice on the full
    HunyuanVideo-like layer: identical lists and outputs."""
    w = WORKLOADS["hunyuan"]
    q, k, v = make_qkv(w)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    del q, k, v
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, micro_heads(w)))
    keys = ("counts", "idx", "m_counts", "m_idx", "o", "lse")
    first = {n: t.clone() for n, t in run(dq, dk, dv).items() if n in keys}
    # scribble over every output between the runs
    for n in keys:
        run.buf[n].fill_(-3)
    second = run(dq, dk, dv)
    assert vsa.read_device_status() == 0
    for n in ("counts", "m_counts"):
        assert torch.equal(first[n], second[n]), n
    for n, cn in (("idx", "counts"), ("m_idx", "m_counts")):
        c = first[cn]
        width = first[n].shape[-1]
        valid = torch.arange(width, device="cuda").view(*([1] * c.dim()), width) < c.unsqueeze(-1)
        assert torch.equal(first[n][valid], second[n][valid]), n
    assert torch.equal(first["o"].view(torch.int16), second["o"].view(torch.int16))
    assert torch.equal(first["lse"].view(torch.int32), second["lse"].view(torch.int32))
