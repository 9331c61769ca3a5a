"""Python binding of libvsa, the B200 block-sparse video attention library.

Argument marshalling only: every step of the path runs in the CUDA kernels of
libvsa.so (built in-tree by ``block_sparse_attention_pool_b200.build``).
PyTorch supplies device memory and the current CUDA stream.  There is no
fallback: if the shared library is missing or cannot be loaded, every call
raises :class:`VsaError`.

Functions mirror the C ABI of ``include/vsa.h`` one to one (same names without
the ``vsa_`` prefix).  :class:`SparseVideoAttention` strings them together into
the whole path (pool -> select -> Macro pass -> Micro select -> Micro pass with
the LSE merge) over caller-visible buffers that it allocates once per shape.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Dict, Optional, Sequence

import torch

__all__ = [
    "VsaError", "Shape", "SelectParams", "MicroParams", "lib", "library_path", "EXPORTED",
    "pool_qk", "select_blocks", "mask_to_lists", "select_micro", "select_micro_workspace_bytes", "select_micro_noalloc",
    "block_sparse_fwd", "lse_merge", "read_device_status", "status_string", "version", "selftest_wait_timeout",
    "PathConfig", "SparseVideoAttention", "ClusterParams", "cluster_count", "cluster_tokens", "permute_rows",
    "select_clusters", "merge_clusters", "merge_clusters_workspace_bytes", "cluster_rows_capacity", "cluster_plan",
    "gather_rows", "cluster_group_fwd", "ClusterBlockConfig", "ClusterBlockAttention",
    "pool_kv_bf16", "rectify_fwd", "SelectionSchedule", "cluster_anchor", "cluster_refine",
    "cluster_refine_workspace_bytes", "subset_size", "PathParams", "path_params", "path_workspace_bytes",
    "path_fwd", "path_host_workspace_bytes", "path_fwd_host", "bind_status_word",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libvsa.so")

EXPORTED = (
    "vsa_status_string", "vsa_version", "vsa_read_device_status", "vsa_bind_status_word", "vsa_pool_qk", "vsa_select_blocks",
    "vsa_mask_to_lists", "vsa_select_micro_workspace_bytes", "vsa_select_micro", "vsa_select_micro_noalloc",
    "vsa_block_sparse_fwd", "vsa_block_sparse_fwd_heads", "vsa_lse_merge", "vsa_selftest_wait_timeout",
    "vsa_selftest_exp2", "vsa_path_workspace_bytes", "vsa_path_fwd", "vsa_path_host_workspace_bytes",
    "vsa_path_fwd_host",
    "vsa_cluster_count", "vsa_cluster_tokens", "vsa_permute_rows", "vsa_select_clusters",
    "vsa_merge_clusters_workspace_bytes", "vsa_merge_clusters", "vsa_cluster_rows_capacity", "vsa_cluster_plan",
    "vsa_gather_rows", "vsa_cluster_group_fwd", "vsa_pool_kv_bf16", "vsa_rectify_fwd", "vsa_cluster_anchor",
    "vsa_cluster_refine_workspace_bytes", "vsa_cluster_refine",
)

STATUS = {0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_UNSUPPORTED", 3: "VSA_ERR_CUDA",
          4: "VSA_ERR_CAPACITY", 5: "VSA_ERR_BAD_INDEX", 6: "VSA_ERR_TIMEOUT", 7: "VSA_ERR_SCRATCH_LIMIT"}

# Fixed scratch of vsa_select_micro_noalloc (include/vsa.h VSA_MICRO_NOALLOC_MAX_BYTES)
MICRO_NOALLOC_MAX_BYTES = 16 << 20


class VsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("n_valid", ctypes.c_int), ("n_pad", ctypes.c_int),
                ("d", ctypes.c_int)]


class ClusterParams(ctypes.Structure):
    """vsa_cluster_params: token lattice, cell extents (tokens), window (cells), rounds."""
    _fields_ = [("lattice_t", ctypes.c_int), ("lattice_h", ctypes.c_int), ("lattice_w", ctypes.c_int),
                ("cell_t", ctypes.c_int), ("cell_h", ctypes.c_int), ("cell_w", ctypes.c_int),
                ("win_t", ctypes.c_int), ("win_h", ctypes.c_int), ("win_w", ctypes.c_int), ("iters", ctypes.c_int)]

    @staticmethod
    def make(lattice, cell, window, iters) -> "ClusterParams":
        return ClusterParams(*[int(v) for v in (*lattice, *cell, *window, iters)])


class SelectParams(ctypes.Structure):
    _fields_ = [("k_min", ctypes.c_int), ("cum_mass", ctypes.c_float), ("fixed_k", ctypes.c_int),
                ("n_anchor", ctypes.c_int), ("anchor_rot", ctypes.c_int)]


class MicroParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("topk", ctypes.c_int), ("percentile", ctypes.c_double),
                ("head_enable", ctypes.POINTER(ctypes.c_uint8)), ("row_capacity", ctypes.c_int)]


class PathParams(ctypes.Structure):
    """vsa_path_params: the whole path's knobs (micro_heads is a HOST array)."""
    _fields_ = [("bq", ctypes.c_int), ("bk", ctypes.c_int), ("scale", ctypes.c_float), ("select", SelectParams),
                ("micro_mode", ctypes.c_int), ("micro_topk", ctypes.c_int), ("micro_percentile", ctypes.c_double),
                ("micro_heads", ctypes.POINTER(ctypes.c_uint8)), ("micro_capacity", ctypes.c_int),
                ("o_fp32", ctypes.c_int)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libvsa.so (once).  Raises VsaError if it is absent: no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise VsaError(3, f"libvsa.so not built at {_LIB_PATH} (run python -m block_sparse_attention_pool_b200.build)")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, F, D, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_size_t
    SP = ctypes.POINTER(Shape)
    L.vsa_status_string.restype = ctypes.c_char_p
    L.vsa_status_string.argtypes = [I]
    L.vsa_version.restype = I
    L.vsa_version.argtypes = []
    L.vsa_read_device_status.restype = I
    L.vsa_read_device_status.argtypes = [P]
    L.vsa_bind_status_word.restype = I
    L.vsa_bind_status_word.argtypes = [P, P]
    L.vsa_selftest_wait_timeout.restype = I
    L.vsa_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, P]
    L.vsa_selftest_exp2.restype = I
    L.vsa_selftest_exp2.argtypes = [P, P, ctypes.c_int, P]
    L.vsa_pool_qk.restype = I
    L.vsa_pool_qk.argtypes = [P, P, SP, I, I, P, P, P, P, P]
    L.vsa_select_blocks.restype = I
    L.vsa_select_blocks.argtypes = [P, P, SP, I, I, F, ctypes.POINTER(SelectParams), P, P, P, P]
    L.vsa_mask_to_lists.restype = I
    L.vsa_mask_to_lists.argtypes = [P, SP, I, I, P, P, P]
    L.vsa_select_micro_workspace_bytes.restype = S
    L.vsa_select_micro_workspace_bytes.argtypes = [SP, ctypes.POINTER(MicroParams)]
    L.vsa_select_micro.restype = I
    L.vsa_select_micro.argtypes = [P, P, P, P, SP, I, I, F, ctypes.POINTER(MicroParams), P, P, P, S, P]
    L.vsa_select_micro_noalloc.restype = I
    L.vsa_select_micro_noalloc.argtypes = [P, P, P, P, SP, I, I, F, ctypes.POINTER(MicroParams), P, P, P]
    L.vsa_block_sparse_fwd.restype = I
    L.vsa_block_sparse_fwd.argtypes = [P, P, P, SP, I, I, P, P, I, F, P, I, P, P, P, P]
    L.vsa_block_sparse_fwd_heads.restype = I
    L.vsa_block_sparse_fwd_heads.argtypes = [P, P, P, SP, I, I, P, P, I, F, P, I, P, P, P, P, I, P]
    L.vsa_lse_merge.restype = I
    L.vsa_lse_merge.argtypes = [P, P, P, P, SP, P, I, P, P]
    L.vsa_cluster_count.restype = I
    L.vsa_cluster_count.argtypes = [ctypes.POINTER(ClusterParams)]
    L.vsa_cluster_tokens.restype = I
    L.vsa_cluster_tokens.argtypes = [P, SP, ctypes.POINTER(ClusterParams), P, P, P, P, P]
    L.vsa_permute_rows.restype = I
    L.vsa_permute_rows.argtypes = [P, P, I, I, I, I, P, P]
    L.vsa_select_clusters.restype = I
    L.vsa_merge_clusters_workspace_bytes.restype = S
    L.vsa_merge_clusters_workspace_bytes.argtypes = [I, I]
    L.vsa_merge_clusters.restype = I
    L.vsa_merge_clusters.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, S, P, P, P, P]
    L.vsa_cluster_rows_capacity.restype = I
    L.vsa_cluster_rows_capacity.argtypes = [I, I]
    L.vsa_cluster_plan.restype = I
    L.vsa_cluster_plan.argtypes = [P, P, P, P, I, I, I, I, I, I, P, P, P, P, P]
    L.vsa_gather_rows.restype = I
    L.vsa_gather_rows.argtypes = [P, P, I, I, I, I, ctypes.c_uint32, P, P]
    L.vsa_cluster_group_fwd.restype = I
    L.vsa_cluster_group_fwd.argtypes = [P, P, P, SP, I, P, P, P, I, P, P, I, F, P, I, P, P]
    L.vsa_cluster_anchor.restype = I
    L.vsa_cluster_anchor.argtypes = [P, SP, ctypes.POINTER(ClusterParams), I, P, P, P, P, P, P, P]
    L.vsa_cluster_refine_workspace_bytes.restype = S
    L.vsa_cluster_refine_workspace_bytes.argtypes = [SP, ctypes.POINTER(ClusterParams)]
    L.vsa_cluster_refine.restype = I
    L.vsa_cluster_refine.argtypes = [P, SP, ctypes.POINTER(ClusterParams), P, I, P, P, P, P, P, S, P]
    L.vsa_pool_kv_bf16.restype = I
    L.vsa_pool_kv_bf16.argtypes = [P, P, SP, I, I, P, P, P]
    PP = ctypes.POINTER(PathParams)
    L.vsa_path_workspace_bytes.restype = S
    L.vsa_path_workspace_bytes.argtypes = [SP, PP]
    L.vsa_path_fwd.restype = I
    L.vsa_path_fwd.argtypes = [P, P, P, SP, PP, P, P, P, S, P]
    L.vsa_path_host_workspace_bytes.restype = S
    L.vsa_path_host_workspace_bytes.argtypes = [SP, PP, I]
    L.vsa_path_fwd_host.restype = I
    L.vsa_path_fwd_host.argtypes = [P, P, P, SP, PP, I, P, P, P, S, P]
    L.vsa_rectify_fwd.restype = I
    L.vsa_rectify_fwd.argtypes = [P, P, P, SP, I, I, I, P, P, I, F, P, P, P, I, P, P, I, P]
    L.vsa_select_clusters.argtypes = [P, P, P, P, I, I, I, I, F, ctypes.POINTER(SelectParams), P, P, P]
    _lib = L
    return L


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(code: int, what: str) -> None:
    if code != 0:
        raise VsaError(code, what)


def _shape(B, H, n_valid, n_pad, d) -> Shape:
    return Shape(int(B), int(H), int(n_valid), int(n_pad), int(d))


def shape_of(q: torch.Tensor, n_valid: int) -> Shape:
    B, H, n_pad, d = q.shape
    return _shape(B, H, n_valid, n_pad, d)


def status_string(code: int) -> str:
    return lib().vsa_status_string(int(code)).decode()


def version() -> int:
    return lib().vsa_version()


def read_device_status(stream=None) -> int:
    return lib().vsa_read_device_status(_s(stream))


def bind_status_word(word: Optional[torch.Tensor], stream=None) -> None:
    """Make the calls later enqueued on ``stream`` report device-side errors
    into ``word`` (a device int32 tensor of 2 elements, cleared here) instead
    of the process-wide word; None removes the binding.  read_device_status
    on that stream then reads (and clears) ``word``."""
    if word is not None and (not word.is_cuda or word.dtype != torch.int32 or word.numel() < 2):
        raise ValueError("the status word is a device int32 tensor of at least 2 elements")
    _check(lib().vsa_bind_status_word(_s(stream), _p(word)), "vsa_bind_status_word")


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test (a wait nothing completes, given up
    after limit_ns); the device status then reads VSA_ERR_TIMEOUT."""
    _check(lib().vsa_selftest_wait_timeout(int(limit_ns), _s(stream)), "vsa_selftest_wait_timeout")


def selftest_exp2(x: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """y = 2**x by the exponential the attention softmax runs on the FMA pipe
    for part of its logits (x, y: contiguous fp32 device tensors of one size)."""
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise ValueError("x and y must be fp32 tensors of the same size")
    if not (x.is_contiguous() and y.is_contiguous()):
        raise ValueError("x and y must be contiguous")
    _check(lib().vsa_selftest_exp2(_p(x), _p(y), int(x.numel()), _s(stream)), "vsa_selftest_exp2")


def pool_qk(q, k, shape: Shape, bq, bk, q_pool, k_pool, q_pool64=None, k_pool16=None, stream=None):
    _check(lib().vsa_pool_qk(_p(q), _p(k), ctypes.byref(shape), bq, bk, _p(q_pool), _p(k_pool), _p(q_pool64),
                             _p(k_pool16), _s(stream)), "vsa_pool_qk")


def select_blocks(q_pool, k_pool, shape: Shape, bq, bk, scale, params: SelectParams, counts, idx, mask=None,
                  stream=None):
    _check(lib().vsa_select_blocks(_p(q_pool), _p(k_pool), ctypes.byref(shape), bq, bk, float(scale),
                                   ctypes.byref(params), _p(counts), _p(idx), _p(mask), _s(stream)),
           "vsa_select_blocks")


def select_clusters(mu_q, mu_k, sizes_q, sizes_k, scale, params: SelectParams, counts, idx, stream=None):
    """Cluster-level selection; mu_* fp32 [B, H, n, d], sizes_* int32 [B, H, n]."""
    bh = mu_q.shape[0] * mu_q.shape[1]
    _check(lib().vsa_select_clusters(_p(mu_q), _p(mu_k), _p(sizes_q), _p(sizes_k), bh, mu_q.shape[2],
                                     mu_k.shape[2], mu_q.shape[3], float(scale), ctypes.byref(params), _p(counts),
                                     _p(idx), _s(stream)), "vsa_select_clusters")


def merge_clusters_workspace_bytes(batch_heads: int, n_q: int) -> int:
    return int(lib().vsa_merge_clusters_workspace_bytes(batch_heads, n_q))


def merge_clusters(sizes_q, sizes_k, counts, idx, sides, tau_q, tau_k, workspace, group_of, g_counts, g_idx,
                   stream=None):
    """Algorithm 1 merging; sizes_* int32 [B, H, n], sides uint8 [B, H, R, n_q]
    (or None for R = 0), workspace a uint8 device buffer."""
    bh = sizes_q.shape[0] * sizes_q.shape[1]
    rounds = 0 if sides is None else sides.shape[2]
    _check(lib().vsa_merge_clusters(_p(sizes_q), _p(sizes_k), _p(counts), _p(idx), _p(sides), bh, sizes_q.shape[2],
                                    sizes_k.shape[2], rounds, int(tau_q), int(tau_k), _p(workspace),
                                    workspace.numel() * workspace.element_size(), _p(group_of), _p(g_counts),
                                    _p(g_idx), _s(stream)), "vsa_merge_clusters")


def cluster_rows_capacity(n_valid: int, n_q: int) -> int:
    return int(lib().vsa_cluster_rows_capacity(n_valid, n_q))


def cluster_plan(group_of, sizes_q, perm_q, sizes_k, n_valid, qmap, qinv, tile_list, kc_off, stream=None):
    """Query-layout plan of the groups; group_of/sizes_* int32 [B, H, n], perm_q
    int32 [B, H, n_pad], qmap [B, H, n_rows], qinv [B, H, n_pad], tile_list
    [B, H, n_rows/128], kc_off [B, H, n_k]."""
    B, H, nq = sizes_q.shape
    _check(lib().vsa_cluster_plan(_p(group_of), _p(sizes_q), _p(perm_q), _p(sizes_k), B * H, nq, sizes_k.shape[2],
                                  int(n_valid), perm_q.shape[2], qmap.shape[2], _p(qmap), _p(qinv), _p(tile_list),
                                  _p(kc_off), _s(stream)), "vsa_cluster_plan")


def gather_rows(src, mp, dst, fill: int = 0, stream=None):
    """dst[b, h, i] = src[b, h, mp[b, h, i]] (-1: fill word, -2: untouched); rows
    are the trailing dimensions after [B, H, n]."""
    B, H, n_src = src.shape[:3]
    n_dst = dst.shape[2]
    row_bytes = (src.numel() // (B * H * n_src)) * src.element_size()
    _check(lib().vsa_gather_rows(_p(src), _p(mp), B * H, n_src, n_dst, row_bytes, ctypes.c_uint32(fill & 0xffffffff),
                                 _p(dst), _s(stream)), "vsa_gather_rows")


def cluster_group_fwd(q_rows, k, v, shape: Shape, tile_list, kc_off, kc_size, counts, idx, scale, o, lse,
                      stream=None):
    """Attention of the query layout's tiles to their groups' key clusters."""
    n_rows = q_rows.shape[2]
    _check(lib().vsa_cluster_group_fwd(_p(q_rows), _p(k), _p(v), ctypes.byref(shape), n_rows, _p(tile_list),
                                       _p(kc_off), _p(kc_size), kc_size.shape[2], _p(counts), _p(idx),
                                       counts.shape[2], float(scale), _p(o), 1 if o.dtype == torch.float32 else 0,
                                       _p(lse), _s(stream)), "vsa_cluster_group_fwd")


def pool_kv_bf16(k, v, shape: Shape, bk, k_bar, v_bar, stream=None):
    """bf16 block means of K and V: k_bar, v_bar [B, H, n_rows, d]."""
    _check(lib().vsa_pool_kv_bf16(_p(k), _p(v), ctypes.byref(shape), bk, k_bar.shape[2], _p(k_bar), _p(v_bar),
                                  _s(stream)), "vsa_pool_kv_bf16")


def rectify_fwd(q, k_bar, v_bar, shape: Shape, bq, bk, counts, idx, idx_stride, scale, o, lse, merge_o=None,
                merge_lse=None, heads=None, stream=None):
    """Pooled pass over the omitted blocks, merged into (merge_o, merge_lse)."""
    if heads is None:
        hp, nh = None, shape.B * shape.H
    else:
        hp, nh = _p(heads), heads.numel()
    _check(lib().vsa_rectify_fwd(_p(q), _p(k_bar), _p(v_bar), ctypes.byref(shape), bq, bk, k_bar.shape[2],
                                 _p(counts), _p(idx), idx_stride, float(scale), _p(merge_o), _p(merge_lse), _p(o),
                                 1 if o.dtype == torch.float32 else 0, _p(lse), hp, nh, _s(stream)),
           "vsa_rectify_fwd")


def subset_size(n_valid: int, frac: float) -> int:
    """ceil(frac * n_valid): the cached subset of the hybrid clustering."""
    return int(math.ceil(frac * n_valid))


def cluster_anchor(x, shape: Shape, params: "ClusterParams", assign, centroids, sizes, perm, ratio, subset,
                   stream=None):
    """Anchor step: full clustering plus Lowe's ratio and the cached subset
    (subset int32 [B, H, n_sub])."""
    _check(lib().vsa_cluster_anchor(_p(x), ctypes.byref(shape), ctypes.byref(params), subset.shape[2], _p(assign),
                                    _p(centroids), _p(sizes), _p(perm), _p(ratio), _p(subset), _s(stream)),
           "vsa_cluster_anchor")


def cluster_refine_workspace_bytes(shape: Shape, params: "ClusterParams") -> int:
    return int(lib().vsa_cluster_refine_workspace_bytes(ctypes.byref(shape), ctypes.byref(params)))


def cluster_refine(x, shape: Shape, params: "ClusterParams", subset, assign, centroids, sizes, perm, workspace,
                   stream=None):
    """Intermediate step: global reassignment of the cached subset, update of the
    touched centroids, sizes and permutation rebuilt (assign, centroids in place)."""
    _check(lib().vsa_cluster_refine(_p(x), ctypes.byref(shape), ctypes.byref(params), _p(subset), subset.shape[2],
                                    _p(assign), _p(centroids), _p(sizes), _p(perm), _p(workspace),
                                    workspace.numel() * workspace.element_size(), _s(stream)), "vsa_cluster_refine")


def mask_to_lists(mask, shape: Shape, bq, bk, counts, idx, stream=None):
    _check(lib().vsa_mask_to_lists(_p(mask), ctypes.byref(shape), bq, bk, _p(counts), _p(idx), _s(stream)),
           "vsa_mask_to_lists")


def _micro_params(mode, topk, percentile, head_enable: Optional[Sequence[int]], row_capacity):
    arr = None
    if head_enable is not None:
        arr = (ctypes.c_uint8 * len(head_enable))(*[int(x) for x in head_enable])
    p = MicroParams(int(mode), int(topk), float(percentile),
                    ctypes.cast(arr, ctypes.POINTER(ctypes.c_uint8)) if arr is not None else None,
                    int(row_capacity))
    return p, arr  # keep arr alive with p


def select_micro_workspace_bytes(shape: Shape, mode, topk, percentile, head_enable, row_capacity) -> int:
    p, keep = _micro_params(mode, topk, percentile, head_enable, row_capacity)
    n = lib().vsa_select_micro_workspace_bytes(ctypes.byref(shape), ctypes.byref(p))
    del keep
    return int(n)


def select_micro(q_pool64, k_pool16, counts, idx, shape: Shape, bq, bk, scale, mode, topk, percentile, head_enable,
                 row_capacity, m_counts, m_idx, workspace, stream=None):
    p, keep = _micro_params(mode, topk, percentile, head_enable, row_capacity)
    _check(lib().vsa_select_micro(_p(q_pool64), _p(k_pool16), _p(counts), _p(idx), ctypes.byref(shape), bq, bk,
                                  float(scale), ctypes.byref(p), _p(m_counts), _p(m_idx), _p(workspace),
                                  workspace.numel() * workspace.element_size(), _s(stream)), "vsa_select_micro")
    del keep


def select_micro_noalloc(q_pool64, k_pool16, counts, idx, shape: Shape, bq, bk, scale, mode, topk, percentile,
                         head_enable, row_capacity, m_counts, m_idx, stream=None):
    """vsa_select_micro without a workspace argument: for callers that may not
    allocate device memory themselves (its scratch is the library's fixed
    array of MICRO_NOALLOC_MAX_BYTES per GPU; calls must not overlap on the GPU)."""
    p, keep = _micro_params(mode, topk, percentile, head_enable, row_capacity)
    _check(lib().vsa_select_micro_noalloc(_p(q_pool64), _p(k_pool16), _p(counts), _p(idx), ctypes.byref(shape), bq,
                                          bk, float(scale), ctypes.byref(p), _p(m_counts), _p(m_idx), _s(stream)),
           "vsa_select_micro_noalloc")
    del keep


def block_sparse_fwd(q, k, v, shape: Shape, list_rows, seg_keys, counts, idx, idx_stride, scale, o, lse,
                     merge_o=None, merge_lse=None, stream=None, heads=None):
    """``heads``: None (every (batch, head)) or a device int32 tensor of
    flattened indices b*H + h; only those heads are read and written."""
    o_fp32 = 1 if o.dtype == torch.float32 else 0
    if heads is None:
        _check(lib().vsa_block_sparse_fwd(_p(q), _p(k), _p(v), ctypes.byref(shape), int(list_rows), int(seg_keys),
                                          _p(counts), _p(idx), int(idx_stride), float(scale), _p(o), o_fp32, _p(lse),
                                          _p(merge_o), _p(merge_lse), _s(stream)), "vsa_block_sparse_fwd")
        return
    if heads.dtype != torch.int32 or not heads.is_contiguous():
        raise ValueError("heads must be a contiguous int32 tensor")
    _check(lib().vsa_block_sparse_fwd_heads(_p(q), _p(k), _p(v), ctypes.byref(shape), int(list_rows),
                                            int(seg_keys), _p(counts), _p(idx), int(idx_stride), float(scale), _p(o),
                                            o_fp32, _p(lse), _p(merge_o), _p(merge_lse), _p(heads),
                                            int(heads.numel()), _s(stream)), "vsa_block_sparse_fwd_heads")


def cluster_count(params: ClusterParams) -> int:
    return int(lib().vsa_cluster_count(ctypes.byref(params)))


def cluster_tokens(x, shape: Shape, params: ClusterParams, assign, centroids, sizes, perm, stream=None):
    _check(lib().vsa_cluster_tokens(_p(x), ctypes.byref(shape), ctypes.byref(params), _p(assign), _p(centroids),
                                    _p(sizes), _p(perm), _s(stream)), "vsa_cluster_tokens")


def permute_rows(src, perm, dst, inverse: bool = False, stream=None):
    """Rows of src [B, H, n_pad, ...] gathered by perm [B, H, n_pad] into dst
    (inverse: scattered)."""
    B, H, n_pad = perm.shape
    row_bytes = src[0, 0, 0].numel() * src.element_size() if src.dim() > 3 else src.element_size()
    _check(lib().vsa_permute_rows(_p(src), _p(perm), B * H, n_pad, row_bytes, 1 if inverse else 0, _p(dst),
                                  _s(stream)), "vsa_permute_rows")


def lse_merge(o_a, lse_a, o_b, lse_b, shape: Shape, o_out, lse_out, stream=None):
    out_fp32 = 1 if o_out.dtype == torch.float32 else 0
    _check(lib().vsa_lse_merge(_p(o_a), _p(lse_a), _p(o_b), _p(lse_b), ctypes.byref(shape), _p(o_out), out_fp32,
                               _p(lse_out), _s(stream)), "vsa_lse_merge")


# ---------------------------------------------------------------------------
# The whole path
# ---------------------------------------------------------------------------

def path_params(cfg: "PathConfig", micro_heads=None, o_fp32: bool = False):
    """vsa_path_params of a PathConfig (token-order layout, no rectification).
    Returns (params, keep): keep holds the host flag array alive."""
    if cfg.rectify or cfg.cluster_lattice is not None:
        raise ValueError("the one-call path covers pooling, selection, Macro and Micro passes only")
    flags = cfg.micro_heads if micro_heads is None else micro_heads
    arr = None
    if cfg.micro_mode and flags is not None:
        arr = (ctypes.c_uint8 * len(flags))(*[int(x) for x in flags])
    p = PathParams(int(cfg.bq), int(cfg.bk), float(cfg.scale or 0.0),
                   SelectParams(cfg.k_min, cfg.cum_mass, cfg.fixed_k, cfg.n_anchor, cfg.anchor_rot),
                   int(cfg.micro_mode), int(cfg.micro_topk), float(cfg.micro_percentile),
                   ctypes.cast(arr, ctypes.POINTER(ctypes.c_uint8)) if arr is not None else None,
                   int(cfg.micro_capacity), 1 if o_fp32 else 0)
    return p, arr


def path_workspace_bytes(shape: Shape, params: PathParams) -> int:
    return int(lib().vsa_path_workspace_bytes(ctypes.byref(shape), ctypes.byref(params)))


def path_fwd(q, k, v, shape: Shape, params: PathParams, o, lse, workspace, stream=None):
    """The whole path in one C call on device tensors."""
    _check(lib().vsa_path_fwd(_p(q), _p(k), _p(v), ctypes.byref(shape), ctypes.byref(params), _p(o), _p(lse),
                              _p(workspace), workspace.numel() * workspace.element_size(), _s(stream)),
           "vsa_path_fwd")


def path_host_workspace_bytes(shape: Shape, params: PathParams, chunk_heads: int) -> int:
    return int(lib().vsa_path_host_workspace_bytes(ctypes.byref(shape), ctypes.byref(params), int(chunk_heads)))


def path_fwd_host(q_h, k_h, v_h, shape: Shape, params: PathParams, chunk_heads: int, o_h, lse_h, workspace,
                  stream=None):
    """The whole path in one C call on HOST tensors (pinned), the copies
    pipelined over chunks of heads; complete when ``stream`` is."""
    for t in (q_h, k_h, v_h, o_h, lse_h):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("path_fwd_host takes contiguous host tensors")
    _check(lib().vsa_path_fwd_host(_p(q_h), _p(k_h), _p(v_h), ctypes.byref(shape), ctypes.byref(params),
                                   int(chunk_heads), _p(o_h), _p(lse_h), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _s(stream)),
           "vsa_path_fwd_host")


@dataclass
class PathConfig:
    """Sizes and knobs of one attention layer (field names as in vsa.h)."""
    n_valid: int
    bq: int = 128
    bk: int = 128
    scale: Optional[float] = None
    k_min: int = 0
    cum_mass: float = 0.0
    fixed_k: int = 0
    n_anchor: int = 0
    anchor_rot: int = 0
    micro_mode: int = 0
    micro_topk: int = 0
    micro_percentile: float = 0.0
    micro_heads: Optional[Sequence[int]] = None
    micro_capacity: int = 0          # 0: every tile of the row fits (no overflow possible)
    # pooled rectification of the omitted blocks (Rectified SpaAttn; replaces the Micro repair)
    rectify: bool = False
    rectify_heads: Optional[Sequence[int]] = None   # per-head flags; None = every head
    # cluster-permuted layout (HyperVAttention Eq. (1), (4), (5)): None = tokens in their own order
    cluster_lattice: Optional[Sequence[int]] = None   # (T, H, W) with T*H*W == n_valid
    cluster_cell: Sequence[int] = (3, 5, 8)
    cluster_window: Sequence[int] = (3, 5, 5)
    cluster_iters: int = 3

    def cluster_params(self) -> "ClusterParams":
        return ClusterParams.make(self.cluster_lattice, self.cluster_cell, self.cluster_window, self.cluster_iters)

    @staticmethod
    def from_workload(w, micro_heads=None) -> "PathConfig":
        return PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale, k_min=w.k_min, cum_mass=w.cum_mass,
                          fixed_k=w.fixed_k, n_anchor=w.n_anchor, anchor_rot=w.anchor_rot, micro_mode=w.micro_mode,
                          micro_topk=w.micro_topk, micro_percentile=w.micro_percentile,
                          micro_heads=None if micro_heads is None else [int(x) for x in micro_heads])


class SparseVideoAttention:
    """Pool -> select -> Macro attention -> Micro select -> Micro attention + LSE merge.

    Buffers are allocated once per input shape (torch, on q's device) and
    reused; outputs of the last call stay readable in ``self.buf``.
    """

    def __init__(self, cfg: PathConfig, workspace_for_all_heads: bool = False):
        self.cfg = cfg
        self.buf: Dict[str, torch.Tensor] = {}
        self._key = None
        self._selected = None  # shape of the last call that ran selection
        # size the Micro workspace as if every head were enabled (callers that
        # pass different per-call head flags)
        self._ws_all = workspace_for_all_heads

    def _alloc(self, q: torch.Tensor):
        B, H, n_pad, d = q.shape
        key = (B, H, n_pad, d, q.device)
        if key == self._key:
            return
        self._selected = None
        c = self.cfg
        dev = q.device
        n_q, n_k = n_pad // c.bq, n_pad // c.bk
        f32, i32 = torch.float32, torch.int32
        b = {
            "q_pool": torch.empty(B, H, n_q, d, device=dev, dtype=f32),
            "k_pool": torch.empty(B, H, n_k, d, device=dev, dtype=f32),
            "counts": torch.empty(B, H, n_q, device=dev, dtype=i32),
            "idx": torch.empty(B, H, n_q, n_k, device=dev, dtype=i32),
            "lse": torch.empty(B, H, n_pad, device=dev, dtype=f32),
            "o": torch.empty(B, H, n_pad, d, device=dev, dtype=torch.bfloat16),
        }
        if c.micro_mode:
            n_r, n_t = n_pad // 64, n_pad // 16
            cap = c.micro_capacity or n_t
            shape = _shape(B, H, c.n_valid, n_pad, d)
            ws = select_micro_workspace_bytes(shape, c.micro_mode, c.micro_topk, c.micro_percentile,
                                              None if self._ws_all else c.micro_heads, cap)
            b.update({
                "q_pool64": torch.empty(B, H, n_r, d, device=dev, dtype=f32),
                "k_pool16": torch.empty(B, H, n_t, d, device=dev, dtype=f32),
                "o_macro": torch.empty(B, H, n_pad, d, device=dev, dtype=f32),
                "lse_macro": torch.empty(B, H, n_pad, device=dev, dtype=f32),
                "m_counts": torch.empty(B, H, n_r, device=dev, dtype=i32),
                "m_idx": torch.empty(B, H, n_r, cap, device=dev, dtype=i32),
                "workspace": torch.empty(max(16, ws), device=dev, dtype=torch.uint8),
            })
            self.micro_cap = cap
        if c.rectify:
            if c.micro_mode:
                raise ValueError("rectification replaces the Micro repair: set micro_mode = 0")
            n_rows = -(-n_k // 128) * 128
            b.update({
                "k_bar": torch.empty(B, H, n_rows, d, device=dev, dtype=torch.bfloat16),
                "v_bar": torch.empty(B, H, n_rows, d, device=dev, dtype=torch.bfloat16),
                "o_macro": torch.empty(B, H, n_pad, d, device=dev, dtype=f32),
                "lse_macro": torch.empty(B, H, n_pad, device=dev, dtype=f32),
            })
        if c.cluster_lattice is not None:
            G = cluster_count(c.cluster_params())
            if G <= 0:
                raise ValueError("invalid clustering parameters")
            bf = torch.bfloat16
            b.update({
                "qp": torch.empty(B, H, n_pad, d, device=dev, dtype=bf),
                "kp": torch.empty(B, H, n_pad, d, device=dev, dtype=bf),
                "vp": torch.empty(B, H, n_pad, d, device=dev, dtype=bf),
                "op": torch.empty(B, H, n_pad, d, device=dev, dtype=bf),
                "lp": torch.empty(B, H, n_pad, device=dev, dtype=f32),
            })
            for name in ("q", "k"):
                b["assign_" + name] = torch.empty(B, H, c.n_valid, device=dev, dtype=i32)
                b["centroids_" + name] = torch.empty(B, H, G, d, device=dev, dtype=f32)
                b["sizes_" + name] = torch.empty(B, H, G, device=dev, dtype=i32)
                b["perm_" + name] = torch.empty(B, H, n_pad, device=dev, dtype=i32)
        self.buf = b
        self._key = key

    def _head_split(self, B: int, H: int, flags, dev):
        """Device index lists (b*H + h) of the heads without and with the
        repair (Micro or rectification); None stands for "every head", an empty
        tuple for "no head"."""
        key = (B, H, None if flags is None else tuple(int(f) for f in flags), dev)
        cache = self.__dict__.setdefault("_splits", {})
        if key not in cache:
            if flags is None:
                cache[key] = ((), None)
            else:
                if len(flags) != H:
                    raise ValueError(f"{len(flags)} head flags for {H} heads")
                rep = [b * H + h for b in range(B) for h in range(H) if flags[h]]
                plain = [b * H + h for b in range(B) for h in range(H) if not flags[h]]
                as_dev = lambda x: torch.tensor(x, dtype=torch.int32, device=dev) if x else ()
                cache[key] = (None if not rep else as_dev(plain), None if not plain else as_dev(rep))
        return cache[key]

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None, out_o=None, out_lse=None,
                 micro_heads=None, on_stage=None, reuse_selection: bool = False) -> Dict[str, torch.Tensor]:
        """Run the path on device tensors q, k, v [B, H, n_pad, d] (bf16).

        ``reuse_selection``: skip pooling and selection (block and Micro) and
        attend with the lists of the last call that selected (cross-step reuse
        of the mask, see SelectionSchedule).

        With ``cfg.cluster_lattice`` set, Q and K are first clustered per
        (batch, head) by 3D local-window clustering, Q', K', V' are the
        cluster-ordered rows (Eq. (1)), the path below runs on them, and O
        and LSE are put back in token order (Eq. (4)); the permutations stay
        in ``self.buf["perm_q"]`` / ``["perm_k"]``.  Otherwise see _run.
        """
        if self.cfg.cluster_lattice is None:
            return self._run(q, k, v, stream, out_o, out_lse, micro_heads, on_stage, reuse_selection)
        if reuse_selection:
            raise ValueError("reuse_selection applies to the token-order layout")
        self._alloc(q)
        b = self.buf
        B, H, n_pad, d = q.shape
        shape = _shape(B, H, self.cfg.n_valid, n_pad, d)
        params = self.cfg.cluster_params()
        for name, x in (("q", q), ("k", k)):
            cluster_tokens(x, shape, params, b["assign_" + name], b["centroids_" + name], b["sizes_" + name],
                           b["perm_" + name], stream)
        permute_rows(q, b["perm_q"], b["qp"], stream=stream)
        permute_rows(k, b["perm_k"], b["kp"], stream=stream)
        permute_rows(v, b["perm_k"], b["vp"], stream=stream)
        self._run(b["qp"], b["kp"], b["vp"], stream, b["op"], b["lp"], micro_heads, on_stage)
        permute_rows(b["op"], b["perm_q"], b["o"] if out_o is None else out_o, inverse=True, stream=stream)
        permute_rows(b["lp"], b["perm_q"], b["lse"] if out_lse is None else out_lse, inverse=True, stream=stream)
        return b

    def _run(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None, out_o=None, out_lse=None,
             micro_heads=None, on_stage=None, reuse: bool = False) -> Dict[str, torch.Tensor]:
        """Run the whole path on device tensors q, k, v [B, H, n_pad, d] (bf16).

        Outputs go to ``self.buf["o"]`` / ``["lse"]``, or to ``out_o`` /
        ``out_lse`` when given (same shapes).  ``micro_heads`` overrides the
        configured per-head Micro flags (length H).  ``on_stage(i)``, when
        given, is called on the host before the first stage (i = 0) and after
        each stage: pooling 1, selection 2, Macro pass 3, Micro selection 4,
        Micro pass 5 (all enqueued, not completed).

        Heads without the Micro repair get their final output from the Macro
        pass; only heads with it keep a fp32 Macro output, and only they run
        the Micro pass that merges into it.
        """
        c = self.cfg
        self._alloc(q)
        b = self.buf
        B, H, n_pad, d = q.shape
        shape = _shape(B, H, c.n_valid, n_pad, d)
        scale = c.scale if c.scale is not None else 1.0 / math.sqrt(d)
        n_k = n_pad // c.bk
        micro = c.micro_mode != 0
        o = b["o"] if out_o is None else out_o
        lse = b["lse"] if out_lse is None else out_lse
        heads = c.micro_heads if micro_heads is None else micro_heads
        stage = on_stage if on_stage is not None else (lambda i: None)
        stage(0)
        if reuse and self._selected != (B, H, n_pad, d):
            raise ValueError("reuse_selection needs a previous call with fresh selection on this shape")
        if not reuse:
            pool_qk(q, k, shape, c.bq, c.bk, b["q_pool"], b["k_pool"], b.get("q_pool64"), b.get("k_pool16"), stream)
        stage(1)
        if not reuse:
            select_blocks(b["q_pool"], b["k_pool"], shape, c.bq, c.bk, scale,
                          SelectParams(c.k_min, c.cum_mass, c.fixed_k, c.n_anchor, c.anchor_rot), b["counts"],
                          b["idx"], None, stream)
            self._selected = (B, H, n_pad, d)
        stage(2)
        if c.rectify:
            # kept blocks exactly (Macro), then the omitted blocks as pooled keys, merged by LSE
            plain, rep = self._head_split(B, H, c.rectify_heads, q.device)
            if not isinstance(plain, tuple):
                block_sparse_fwd(q, k, v, shape, c.bq, c.bk, b["counts"], b["idx"], n_k, scale, o, lse,
                                 stream=stream, heads=plain)
            if not isinstance(rep, tuple):
                block_sparse_fwd(q, k, v, shape, c.bq, c.bk, b["counts"], b["idx"], n_k, scale, b["o_macro"],
                                 b["lse_macro"], stream=stream, heads=rep)
            stage(3)
            if not isinstance(rep, tuple):
                pool_kv_bf16(k, v, shape, c.bk, b["k_bar"], b["v_bar"], stream)
            stage(4)
            if not isinstance(rep, tuple):
                rectify_fwd(q, b["k_bar"], b["v_bar"], shape, c.bq, c.bk, b["counts"], b["idx"], n_k, scale, o, lse,
                            b["o_macro"], b["lse_macro"], heads=rep, stream=stream)
            stage(5)
            return b
        if not micro:
            block_sparse_fwd(q, k, v, shape, c.bq, c.bk, b["counts"], b["idx"], n_k, scale, o, lse, stream=stream)
            stage(3)
            stage(4)
            stage(5)
            return b
        plain, rep = self._head_split(B, H, heads, q.device)
        if not isinstance(plain, tuple):  # heads whose Macro output is final
            block_sparse_fwd(q, k, v, shape, c.bq, c.bk, b["counts"], b["idx"], n_k, scale, o, lse, stream=stream,
                             heads=plain)
        if not isinstance(rep, tuple):    # heads repaired by the Micro pass keep a fp32 Macro output
            block_sparse_fwd(q, k, v, shape, c.bq, c.bk, b["counts"], b["idx"], n_k, scale, b["o_macro"],
                             b["lse_macro"], stream=stream, heads=rep)
        stage(3)
        if not reuse:
            select_micro(b["q_pool64"], b["k_pool16"], b["counts"], b["idx"], shape, c.bq, c.bk, scale,
                         c.micro_mode, c.micro_topk, c.micro_percentile, heads, self.micro_cap, b["m_counts"],
                         b["m_idx"], b["workspace"], stream)
        stage(4)
        if not isinstance(rep, tuple):
            block_sparse_fwd(q, k, v, shape, 64, 16, b["m_counts"], b["m_idx"], self.micro_cap, scale, o, lse,
                             b["o_macro"], b["lse_macro"], stream, heads=rep)
        stage(5)
        return b

    def forward_host(self, q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, o_h: torch.Tensor,
                     lse_h: torch.Tensor, chunk_heads: int = 2, device=None) -> None:
        """The whole path on HOST tensors through one C call (vsa_path_fwd_host):
        pinned bf16 q_h, k_h, v_h [B, H, n_pad, d] in, pinned o_h (bf16, same
        shape) and lse_h (fp32 [B, H, n_pad]) out.

        The library cuts the flattened heads into chunks of ``chunk_heads``
        and pipelines them: host-to-device copies of chunk i+1 and
        device-to-host copies of chunk i-1 overlap the path on chunk i.
        Results equal the device path on all heads at once.  Returns once the
        work is complete.
        """
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        B, H, n_pad, d = q_h.shape
        shape = _shape(B, H, self.cfg.n_valid, n_pad, d)
        params, keep = path_params(self.cfg)
        key = (B, H, n_pad, d, dev, chunk_heads)
        if getattr(self, "_host_key", None) != key:
            n = path_host_workspace_bytes(shape, params, chunk_heads)
            if n == 0:
                raise VsaError(1, "vsa_path_host_workspace_bytes")
            self._host_ws = torch.empty(n, device=dev, dtype=torch.uint8)
            self._host_key = key
        with torch.cuda.device(dev):
            stream = torch.cuda.current_stream(dev)
            path_fwd_host(q_h, k_h, v_h, shape, params, chunk_heads, o_h, lse_h, self._host_ws, stream)
            stream.synchronize()
        del keep


@dataclass
class ClusterBlockConfig:
    """Cluster-aligned blocks (HyperVAttention §2 Eq. (1)-(4) on clusters,
    §4.1 Eq. (5), §4.3 Eq. (7)-(10), Algorithm 1)."""
    n_valid: int
    lattice: Sequence[int]            # (T, H, W) with T*H*W == n_valid
    cell: Sequence[int] = (3, 5, 8)
    window: Sequence[int] = (3, 5, 5)
    iters: int = 3
    scale: Optional[float] = None
    k_min: int = 0
    cum_mass: float = 0.0
    fixed_k: int = 0
    rounds: int = 3                   # merging rounds R (App. A.1: 3)
    tau_q: int = 128                  # CTA tile sizes of the cost model (Eq. (7))
    tau_k: int = 128
    hybrid_frac: float = 0.15         # cached share of tokens at anchor steps (App. A.1: 15%)

    def cluster_params(self) -> "ClusterParams":
        return ClusterParams.make(self.lattice, self.cell, self.window, self.iters)


class ClusterBlockAttention:
    """Cluster Q and K -> select key clusters per query cluster -> merge query
    clusters (Algorithm 1) -> group layout -> attention per group tile ->
    output back in token order.  Every stage is a libvsa kernel; buffers are
    allocated once per input shape and stay readable in ``self.buf``."""

    STAGES = ("cluster_qk", "select", "merge", "plan", "gather_in", "attention", "gather_out")

    def __init__(self, cfg: ClusterBlockConfig):
        self.cfg = cfg
        self.buf: Dict[str, torch.Tensor] = {}
        self._key = None

    def _alloc(self, q: torch.Tensor):
        B, H, n_pad, d = q.shape
        key = (B, H, n_pad, d, q.device)
        if key == self._key:
            return
        c = self.cfg
        G = cluster_count(c.cluster_params())
        if G < 1:
            raise VsaError(1, "ClusterBlockAttention: invalid clustering parameters")
        rows = cluster_rows_capacity(c.n_valid, G)
        dev = q.device
        i32, f32 = torch.int32, torch.float32
        b = {}
        for n in ("q", "k"):
            b["assign_" + n] = torch.empty(B, H, c.n_valid, device=dev, dtype=i32)
            b["centroids_" + n] = torch.empty(B, H, G, d, device=dev, dtype=f32)
            b["sizes_" + n] = torch.empty(B, H, G, device=dev, dtype=i32)
            b["perm_" + n] = torch.empty(B, H, n_pad, device=dev, dtype=i32)
        n_sub = subset_size(c.n_valid, c.hybrid_frac)
        shape = _shape(B, H, c.n_valid, n_pad, d)
        for n in ("q", "k"):
            b["ratio_" + n] = torch.empty(B, H, c.n_valid, device=dev, dtype=f32)
            b["subset_" + n] = torch.empty(B, H, max(1, n_sub), device=dev, dtype=i32)
        b["refine_ws"] = torch.empty(cluster_refine_workspace_bytes(shape, c.cluster_params()), device=dev,
                                     dtype=torch.uint8)
        b["counts"] = torch.empty(B, H, G, device=dev, dtype=i32)
        b["idx"] = torch.empty(B, H, G, G, device=dev, dtype=i32)
        b["merge_ws"] = torch.empty(merge_clusters_workspace_bytes(B * H, G), device=dev, dtype=torch.uint8)
        b["group_of"] = torch.empty(B, H, G, device=dev, dtype=i32)
        b["g_counts"] = torch.empty(B, H, G, device=dev, dtype=i32)
        b["g_idx"] = torch.empty(B, H, G, G, device=dev, dtype=i32)
        b["qmap"] = torch.empty(B, H, rows, device=dev, dtype=i32)
        b["qinv"] = torch.empty(B, H, n_pad, device=dev, dtype=i32)
        b["tile_list"] = torch.empty(B, H, rows // 128, device=dev, dtype=i32)
        b["kc_off"] = torch.empty(B, H, G, device=dev, dtype=i32)
        b["q_rows"] = torch.empty(B, H, rows, d, device=dev, dtype=torch.bfloat16)
        b["kp"] = torch.empty(B, H, n_pad, d, device=dev, dtype=torch.bfloat16)
        b["vp"] = torch.empty(B, H, n_pad, d, device=dev, dtype=torch.bfloat16)
        b["o_rows"] = torch.empty(B, H, rows, d, device=dev, dtype=torch.bfloat16)
        b["lse_rows"] = torch.empty(B, H, rows, device=dev, dtype=f32)
        b["o"] = torch.empty(B, H, n_pad, d, device=dev, dtype=torch.bfloat16)
        b["lse"] = torch.empty(B, H, n_pad, device=dev, dtype=f32)
        self.buf = b
        self._key = key
        self._anchored = False

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, sides: Optional[torch.Tensor] = None,
                 stream=None, on_stage=None, cluster_step: str = "full") -> Dict[str, torch.Tensor]:
        """q, k, v: bf16 device tensors [B, H, n_pad, d].  sides: uint8 device
        tensor [B, H, rounds, G] of bipartition bits (the random draws of
        Algorithm 1), or None for no merging.  ``cluster_step``: "full" (3D
        local-window clustering), "anchor" (the same, plus Lowe's ratio and the
        cached subset of the hybrid strategy) or "refine" (an intermediate
        step: only the cached subset is revisited; needs an earlier anchor).
        ``on_stage(i)`` is called on the host before the first stage (i = 0)
        and after each of STAGES."""
        c = self.cfg
        self._alloc(q)
        b = self.buf
        B, H, n_pad, d = q.shape
        shape = _shape(B, H, c.n_valid, n_pad, d)
        scale = c.scale if c.scale is not None else 1.0 / math.sqrt(d)
        stage = on_stage if on_stage is not None else (lambda i: None)
        if cluster_step not in ("full", "anchor", "refine"):
            raise ValueError("cluster_step is 'full', 'anchor' or 'refine'")
        if cluster_step == "refine" and not self._anchored:
            raise ValueError("a refine step needs an earlier anchor step on this shape")
        stage(0)
        params = c.cluster_params()
        for name, x in (("q", q), ("k", k)):
            args = (b["assign_" + name], b["centroids_" + name], b["sizes_" + name], b["perm_" + name])
            if cluster_step == "full":
                cluster_tokens(x, shape, params, *args, stream)
            elif cluster_step == "anchor":
                cluster_anchor(x, shape, params, *args, b["ratio_" + name], b["subset_" + name], stream)
            else:
                cluster_refine(x, shape, params, b["subset_" + name], b["assign_" + name], b["centroids_" + name],
                               b["sizes_" + name], b["perm_" + name], b["refine_ws"], stream)
        if cluster_step == "anchor":
            self._anchored = True
        elif cluster_step == "full":
            self._anchored = False
        stage(1)
        select_clusters(b["centroids_q"], b["centroids_k"], b["sizes_q"], b["sizes_k"], scale,
                        SelectParams(c.k_min, c.cum_mass, c.fixed_k, 0, 0), b["counts"], b["idx"], stream)
        stage(2)
        merge_clusters(b["sizes_q"], b["sizes_k"], b["counts"], b["idx"], sides, c.tau_q, c.tau_k, b["merge_ws"],
                       b["group_of"], b["g_counts"], b["g_idx"], stream)
        stage(3)
        cluster_plan(b["group_of"], b["sizes_q"], b["perm_q"], b["sizes_k"], c.n_valid, b["qmap"], b["qinv"],
                     b["tile_list"], b["kc_off"], stream)
        stage(4)
        gather_rows(q, b["qmap"], b["q_rows"], 0, stream)
        permute_rows(k, b["perm_k"], b["kp"], stream=stream)
        permute_rows(v, b["perm_k"], b["vp"], stream=stream)
        stage(5)
        cluster_group_fwd(b["q_rows"], b["kp"], b["vp"], shape, b["tile_list"], b["kc_off"], b["sizes_k"],
                          b["g_counts"], b["g_idx"], scale, b["o_rows"], b["lse_rows"], stream)
        stage(6)
        gather_rows(b["o_rows"], b["qinv"], b["o"], 0, stream)
        gather_rows(b["lse_rows"], b["qinv"], b["lse"], 0xff800000, stream)
        stage(7)
        return b


class SelectionSchedule:
    """Cross-step reuse of the block mask over denoising steps.

    MOD-DiT (section on linear pattern prediction): sparsity patterns drift
    slowly and piecewise linearly in the mid-late denoising steps, a full
    attention warm-up comes first, and the pattern is refreshed every
    delta-t steps; HyperVAttention section 3: cluster assignments stay stable
    across adjacent steps.  Reading taken here: the first ``warmup`` steps run
    dense attention, the selection runs at step ``warmup`` and every
    ``refresh`` steps after it, and the steps in between attend with the last
    selected lists (no linear prediction of pattern intensities).
    """

    def __init__(self, warmup: int = 0, refresh: int = 2):
        if warmup < 0 or refresh < 1:
            raise ValueError("warmup >= 0 and refresh >= 1")
        self.warmup = warmup
        self.refresh = refresh

    def mode(self, step: int) -> str:
        """'dense', 'select' or 'reuse' for denoising step ``step`` (0-based)."""
        if step < 0:
            raise ValueError("step >= 0")
        if step < self.warmup:
            return "dense"
        return "select" if (step - self.warmup) % self.refresh == 0 else "reuse"
