"""The one-call path entry points against the stage-by-stage path.

vsa_path_fwd chains pooling, selection, the Macro pass, Micro selection and
the Micro pass with the fused merge inside the library; it must give exactly
(bit for bit) what the same entry points give when a caller chains them
(SparseVideoAttention, checked against the oracle in test_gpu_parity).
vsa_path_fwd_host runs the same path on host buffers, chunk by chunk, with
the copies pipelined against the compute: every chunk size must give the
all-heads result bit for bit.  All calls go through the C ABI.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pool_b200 as vsa
from video_inputs import WORKLOADS, make_qkv, micro_heads

from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_pool_b200 import build
    build.build()
    vsa.lib()
    torch.cuda.init()
    yield
    assert vsa.read_device_status() == 0


CASES = {
    "tiny": (WORKLOADS["tiny"], None, None),
    "tiny_b2_p90": (dataclasses.replace(WORKLOADS["tiny"], B=2, micro_mode=2, micro_percentile=0.9, fixed_k=2),
                    None, (1, 0)),
    "wan13b": (WORKLOADS["wan13b"], (0, 3), None),
    "wan14b": (WORKLOADS["wan14b"], (0, 3), None),
    "hunyuan": (WORKLOADS["hunyuan"], (0, 4), (1, 0, 0, 1)),
}


def _case(name):
    w, heads, flags = CASES[name]
    q, k, v = make_qkv(w, heads=heads)
    H = q.shape[1]
    if w.micro_mode and flags is None:
        flags = micro_heads(w)[:H]
    cfg = vsa.PathConfig.from_workload(w, flags)
    return w, cfg, q, k, v


@pytest.mark.parametrize("name", list(CASES))
def test_path_fwd_equals_the_chained_entry_points(name):
    w, cfg, q, k, v = _case(name)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    ref = vsa.SparseVideoAttention(cfg)(dq, dk, dv)
    o_ref, l_ref = ref["o"].clone(), ref["lse"].clone()
    shape = vsa.shape_of(dq, w.n_valid)
    params, keep = vsa.path_params(cfg)
    ws = torch.empty(vsa.path_workspace_bytes(shape, params), dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)                                   # the workspace's content on entry must not matter
    o = torch.full_like(o_ref, float("nan"))
    lse = torch.full_like(l_ref, float("nan"))
    vsa.path_fwd(dq, dk, dv, shape, params, o, lse, ws)
    assert vsa.read_device_status() == 0
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), l_ref.view(torch.int32))
    # fp32 output: the same O before its final rounding to bf16
    params32, keep32 = vsa.path_params(cfg, o_fp32=True)
    o32 = torch.empty(o_ref.shape, dtype=torch.float32, device="cuda")
    vsa.path_fwd(dq, dk, dv, shape, params32, o32, lse, ws)
    assert vsa.read_device_status() == 0
    assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o_ref.view(torch.int16))
    del keep, keep32


@pytest.mark.parametrize("name,chunks", [("tiny_b2_p90", (1, 3, 4)), ("hunyuan", (1, 3)), ("wan14b", (2,))])
def test_path_fwd_host_equals_the_device_path(name, chunks):
    w, cfg, q, k, v = _case(name)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    shape = vsa.shape_of(dq, w.n_valid)
    params, keep = vsa.path_params(cfg)
    ws = torch.empty(vsa.path_workspace_bytes(shape, params), dtype=torch.uint8, device="cuda")
    o_dev = torch.empty_like(dq)
    l_dev = torch.empty(dq.shape[:3], dtype=torch.float32, device="cuda")
    vsa.path_fwd(dq, dk, dv, shape, params, o_dev, l_dev, ws)
    assert vsa.read_device_status() == 0
    o_ref, l_ref = o_dev.cpu(), l_dev.cpu()
    pin = lambda x: torch.from_numpy(x).to(torch.bfloat16).pin_memory()
    qh, kh, vh = pin(q), pin(k), pin(v)
    for chunk in chunks:
        hws = torch.empty(vsa.path_host_workspace_bytes(shape, params, chunk), dtype=torch.uint8, device="cuda")
        oh = torch.full(o_ref.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
        lh = torch.full(l_ref.shape, float("nan"), dtype=torch.float32).pin_memory()
        stream = torch.cuda.Stream()
        vsa.path_fwd_host(qh, kh, vh, shape, params, chunk, oh, lh, hws, stream)
        stream.synchronize()
        assert vsa.read_device_status() == 0
        assert torch.equal(oh.view(torch.int16), o_ref.view(torch.int16)), chunk
        assert torch.equal(lh.view(torch.int32), l_ref.view(torch.int32)), chunk
    del keep
    assert np.isfinite(l_ref.numpy()).any()
