"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before touching the GPU (no CUDA call is
made by any call in this file)."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_pool_b200 as vsa
from block_sparse_attention_pool_b200 import build as vsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsa.h")


@pytest.fixture(scope="module")
def L():
    vsa_build.build()
    return vsa.lib()


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"VSA_API[^;(]*?\b(vsa_\w+)\s*\(", txt)))


def test_header_declares_the_path_entry_points():
    names = _declared()
    for required in ("vsa_pool_qk", "vsa_select_blocks", "vsa_select_micro", "vsa_block_sparse_fwd",
                     "vsa_lse_merge", "vsa_mask_to_lists"):
        assert required in names
    assert set(names) == set(vsa.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert vsa.status_string(0) == "ok"
    assert "timed out" in vsa.status_string(6)
    assert vsa.version() >= 100


def test_host_validation_rejects_bad_arguments(L):
    shape = vsa.Shape(1, 2, 256, 256, 64)
    null = None
    # null tensors
    assert L.vsa_pool_qk(null, null, ctypes.byref(shape), 64, 64, null, null, null, null, null) == 1
    # unsupported head dimension
    bad = vsa.Shape(1, 2, 256, 256, 96)
    fake = ctypes.c_void_p(16)
    assert L.vsa_pool_qk(fake, fake, ctypes.byref(bad), 64, 64, fake, fake, null, null, null) == 1
    # n_pad not a multiple of 128
    bad = vsa.Shape(1, 2, 200, 200, 64)
    assert L.vsa_block_sparse_fwd(fake, fake, fake, ctypes.byref(bad), 128, 128, fake, fake, 2, 0.125, fake, 0,
                                  fake, null, null, null) == 1
    # bad list geometry
    assert L.vsa_block_sparse_fwd(fake, fake, fake, ctypes.byref(shape), 96, 128, fake, fake, 2, 0.125, fake, 0,
                                  fake, null, null, null) == 1
    assert L.vsa_block_sparse_fwd(fake, fake, fake, ctypes.byref(shape), 128, 48, fake, fake, 2, 0.125, fake, 0,
                                  fake, null, null, null) == 1
    # merge output without its LSE
    assert L.vsa_block_sparse_fwd(fake, fake, fake, ctypes.byref(shape), 128, 128, fake, fake, 2, 0.125, fake, 0,
                                  fake, fake, null, null) == 1
    # head subsets: negative or too many entries, or no list with fewer than B*H heads
    fwd_h = L.vsa_block_sparse_fwd_heads
    for heads, n in ((fake, -1), (fake, 3), (null, 1)):
        assert fwd_h(fake, fake, fake, ctypes.byref(shape), 128, 128, fake, fake, 2, 0.125, fake, 0, fake, null,
                     null, heads, n, null) == 1, n
    # an empty head subset enqueues nothing (and needs no device)
    assert fwd_h(fake, fake, fake, ctypes.byref(shape), 128, 128, fake, fake, 2, 0.125, fake, 0, fake, null,
                 null, fake, 0, null) == 0
    # n_valid > n_pad
    bad = vsa.Shape(1, 2, 300, 256, 64)
    assert L.vsa_lse_merge(fake, fake, fake, fake, ctypes.byref(bad), fake, 0, fake, null) == 1
    # too many key blocks for selection (more than 4096)
    big = vsa.Shape(1, 1, 520_000, 4097 * 128, 128)
    params = vsa.SelectParams(1, 0.9, 0, 0, 0)
    assert L.vsa_select_blocks(fake, fake, ctypes.byref(big), 128, 128, 0.1, ctypes.byref(params), fake, fake,
                               null, null) == 2


def test_micro_workspace_query_is_host_only(L):
    shape = vsa.Shape(1, 24, 118_800, 118_912, 128)
    heads = [1 if h in (0, 5, 7, 11, 13, 20) else 0 for h in range(24)]
    n6 = vsa.select_micro_workspace_bytes(shape, 2, 0, 0.99, heads, 7432)
    nall = vsa.select_micro_workspace_bytes(shape, 2, 0, 0.99, None, 7432)
    per_head_keys = (118_912 // 64) * (118_912 // 16) * 4
    assert n6 >= 6 * per_head_keys and nall >= 24 * per_head_keys and nall > n6
    assert vsa.select_micro_workspace_bytes(shape, 1, 0, 0.0, None, 16) == 0      # topk 0 is invalid
    assert vsa.select_micro_workspace_bytes(shape, 2, 0, 1.5, None, 16) == 0      # percentile out of (0, 1)


def test_path_entry_points_validate_on_the_host(L):
    """vsa_path_*: the workspace queries are host-only, grow with the Micro
    repair and with the chunk size, and bad arguments are refused before
    anything is enqueued."""
    shape = vsa.Shape(1, 24, 118_800, 118_912, 128)
    cfg = vsa.PathConfig(n_valid=118_800, fixed_k=186, micro_mode=2, micro_percentile=0.99,
                         micro_heads=[1 if h in (0, 5) else 0 for h in range(24)])
    p_micro, keep = vsa.path_params(cfg)
    p_plain, _ = vsa.path_params(vsa.PathConfig(n_valid=118_800, fixed_k=186))
    n_micro = vsa.path_workspace_bytes(shape, p_micro)
    n_plain = vsa.path_workspace_bytes(shape, p_plain)
    o_macro = 24 * 118_912 * 128 * 4
    assert n_plain > 0 and n_micro > n_plain + o_macro
    h1 = vsa.path_host_workspace_bytes(shape, p_micro, 1)
    h2 = vsa.path_host_workspace_bytes(shape, p_micro, 2)
    assert 0 < h1 < h2 < n_micro
    assert vsa.path_host_workspace_bytes(shape, p_micro, 0) == 0
    bad = vsa.PathParams.from_buffer_copy(p_plain)
    bad.bq = 96
    assert vsa.path_workspace_bytes(shape, bad) == 0
    fake, null = ctypes.c_void_p(256), None
    assert L.vsa_path_fwd(fake, fake, fake, ctypes.byref(shape), ctypes.byref(bad), fake, fake, fake, 1 << 40,
                          null) == 1
    # workspace too small, misaligned workspace, null output
    assert L.vsa_path_fwd(fake, fake, fake, ctypes.byref(shape), ctypes.byref(p_plain), fake, fake, fake,
                          n_plain - 1, null) == 1
    assert L.vsa_path_fwd(fake, fake, fake, ctypes.byref(shape), ctypes.byref(p_plain), fake, fake,
                          ctypes.c_void_p(272), n_plain, null) == 1
    assert L.vsa_path_fwd_host(fake, fake, fake, ctypes.byref(shape), ctypes.byref(p_plain), 2, null, fake, fake,
                               1 << 40, null) == 1
    del keep


def test_status_word_binding_checks_alignment_on_the_host(L):
    """A status word must be 4-byte aligned device memory; a misaligned one is
    refused before any CUDA call (VSA_ERR_INVALID_ARG)."""
    assert L.vsa_bind_status_word(None, ctypes.c_void_p(0x1002)) == 1
    assert L.vsa_bind_status_word(None, ctypes.c_void_p(0x1001)) == 1
