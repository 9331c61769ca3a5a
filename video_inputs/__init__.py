"""Seeded synthetic video-DiT attention inputs and the workload table.

This module is shared by the CPU oracle and by the CUDA path's tests and
benchmark.  It holds no arithmetic of the attention method itself: it only
draws Q/K/V tensors, rounds them to bfloat16-representable values, and states
the per-workload sizes and selection knobs.

Workloads (token counts from the HyperVAttention page, §5 "Experimental
Settings": 21x45x80 = 75,600 and 33x45x80 = 118,800 tokens at 720p; the
Wan-2.1 480p grid 21x30x52 = 32,760 tokens):

  tiny      B1 H2  d64  grid 4x8x8    (N=256)     blocks 64x64,  top-2 U cum-mass 0.9, Micro top-4 16-key tiles
  wan13b    B1 H12 d128 grid 21x30x52 (N=32,760)  blocks 128x128, cum-mass 0.95 (k_min 1)
  wan14b    B1 H40 d128 grid 21x45x80 (N=75,600, padded to 75,776 as the workload states, so the
            last key block holds no valid key)  blocks 128x128, fixed 15% (k=89) + 2 rotating anchor columns
  hunyuan   B1 H24 d128 grid 33x45x80 (N=118,800) blocks 128x128, fixed 20% (k=186); Micro in 25% of heads,
            64x16 tiles above the 99th percentile of omitted-tile scores; heavy-tailed Q/K
  sweep     the hunyuan tensors, kept fraction in {1, .5, .25, .15, .08} x blocks {128x128, 64x128}

Generators:
  * tiny field: standard-normal tokens + 0.5 x a smooth 3-D positional field,
    the sum of 8 sinusoids over (t, y, x) with integer frequencies in [0, 2]
    cycles per axis extent, uniform phases, and a N(0, 1/8) direction in R^d
    per sinusoid.  The same field is added to Q, K and V of every head.
  * locality field: per frame t a rank-16 matrix U_t W (U_t = low-frequency
    spatial cosines over (y, x), 0 or 1 cycle per axis extent, drawn per
    frame; W ~ N(0, 1/16) the head's feature basis), frames chained so that
    the correlation of frames t and t' is exp(-|t - t'| / 3), scaled to unit
    RMS per element.  Q and K of a head share one field; V gets an
    independent draw.
    Tokens = N(0, 1) + 0.8 x field.
  * heavy tail: 1% of token positions (chosen by seed, same for all heads)
    scaled by 4 in Q and K.

Padding rows (N_valid <= row < N_pad) are zero.  Every tensor is returned as
float32 holding exactly representable bfloat16 values, shape [B, H, N_pad, d].
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Optional, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "sweep_points", "make_qkv", "round_to_bf16",
    "bf16_bits", "micro_heads", "pad_to",
]


def pad_to(n: int, multiple: int) -> int:
    return ((n + multiple - 1) // multiple) * multiple


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: Tuple[int, int, int]          # (T, Y, X) video token grid
    bq: int                             # query block rows
    bk: int                             # key block rows
    seed: int
    generator: str                      # "tiny" | "locality"
    field_scale: float
    heavy_tail: bool = False
    # block selection knobs
    k_min: int = 0                      # top-k floor (union with top-p)
    cum_mass: float = 0.0               # top-p threshold; <= 0 disables
    fixed_k: int = 0                    # > 0: keep exactly this many blocks per row
    n_anchor: int = 0                   # rotating global anchor key-block columns
    anchor_rot: int = 0                 # rotation offset of the anchors
    # Micro knobs
    micro_mode: int = 0                 # 0 off, 1 top-k per micro row, 2 per-head percentile
    micro_topk: int = 0
    micro_percentile: float = 0.0
    micro_head_frac: float = 1.0        # fraction of heads with Micro repair (mode 2)
    micro_rows: int = 64                # query rows per Micro row
    micro_keys: int = 16                # keys per Micro tile
    n_pad_fixed: int = 0                # > 0: padded length stated by the workload

    @property
    def n_valid(self) -> int:
        t, y, x = self.grid
        return t * y * x

    @property
    def n_pad(self) -> int:
        if self.n_pad_fixed:
            return self.n_pad_fixed
        return pad_to(self.n_valid, max(self.bq, self.bk, 128))

    @property
    def n_q(self) -> int:
        return self.n_pad // self.bq

    @property
    def n_k(self) -> int:
        return self.n_pad // self.bk

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_blocks(self, bq: int, bk: int, fixed_k: int) -> "Workload":
        return dataclasses.replace(self, bq=bq, bk=bk, fixed_k=fixed_k, name=f"{self.name}-{bq}x{bk}-k{fixed_k}")


def _fixed_k(frac: float, n_k: int) -> int:
    return min(n_k, max(1, round_half_up(frac * n_k)))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, (4, 8, 8), 64, 64, seed=0, generator="tiny", field_scale=0.5,
                     k_min=2, cum_mass=0.9, micro_mode=1, micro_topk=4),
    "wan13b": Workload("wan13b", 1, 12, 128, (21, 30, 52), 128, 128, seed=1, generator="locality",
                       field_scale=0.8, k_min=1, cum_mass=0.95),
    "wan14b": Workload("wan14b", 1, 40, 128, (21, 45, 80), 128, 128, seed=2, generator="locality",
                       field_scale=0.8, fixed_k=_fixed_k(0.15, 592), n_anchor=2, anchor_rot=2,
                       n_pad_fixed=75_776),
    "hunyuan": Workload("hunyuan", 1, 24, 128, (33, 45, 80), 128, 128, seed=3, generator="locality",
                        field_scale=0.8, heavy_tail=True, fixed_k=_fixed_k(0.20, 929),
                        micro_mode=2, micro_percentile=0.99, micro_head_frac=0.25),
}

SWEEP_FRACTIONS = (1.0, 0.5, 0.25, 0.15, 0.08)
SWEEP_BLOCKS = ((128, 128), (64, 128))


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def sweep_points():
    """The sparsity sweep on the hunyuan tensors: (fraction, Workload) pairs."""
    base = WORKLOADS["hunyuan"]
    pts = []
    for bq, bk in SWEEP_BLOCKS:
        for f in SWEEP_FRACTIONS:
            n_k = base.n_pad // bk
            w = dataclasses.replace(base, bq=bq, bk=bk, fixed_k=_fixed_k(f, n_k), micro_mode=0,
                                    name=f"sweep-{bq}x{bk}-{int(round(f * 100))}pct")
            pts.append((f, w))
    return pts


# ---------------------------------------------------------------------------
# bfloat16 rounding (round to nearest, ties to even) of float32 arrays
# ---------------------------------------------------------------------------

def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Return float32 values exactly representable in bfloat16 (RNE)."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    u = x.view(np.uint32)
    lsb = np.right_shift(u, 16)
    np.bitwise_and(lsb, 1, out=lsb)
    u += np.uint32(0x7FFF)
    u += lsb
    np.bitwise_and(u, np.uint32(0xFFFF0000), out=u)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Fields
# ---------------------------------------------------------------------------

def _coords(grid):
    T, Y, X = grid
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    return t.reshape(-1), y.reshape(-1), x.reshape(-1)


def _tiny_field(rng: np.random.Generator, grid, d: int) -> np.ndarray:
    T, Y, X = grid
    t, y, x = _coords(grid)
    field = np.zeros((t.size, d), dtype=np.float64)
    for _ in range(8):
        ft, fy, fx = rng.integers(0, 3, size=3)
        phase = rng.uniform(0.0, 2.0 * math.pi)
        direction = rng.normal(0.0, math.sqrt(1.0 / 8.0), size=d)
        arg = 2.0 * math.pi * (ft * t / T + fy * y / Y + fx * x / X) + phase
        field += np.sin(arg)[:, None] * direction[None, :]
    return field.astype(np.float32)


def _locality_field(rng: np.random.Generator, grid, d: int, rank: int = 16, tau: float = 3.0,
                    max_freq: int = 1) -> np.ndarray:
    """Rank-16 video locality field of one head, [T*Y*X, d] float32.

    Frame t carries U_t W: U_t [Y*X, rank] are spatial cosines with integer
    frequencies in [0, max_freq] cycles per axis extent and uniform phases (a
    fresh draw per frame), W [rank, d] ~ N(0, 1/rank) is the head's shared
    feature basis.  Frames are chained as an AR(1) sequence with coefficient
    exp(-1/tau), so the correlation of frames t and t' decays as
    exp(-|t - t'| / tau).  The result is scaled to unit RMS per element.
    """
    T, Y, X = grid
    yy, xx = np.meshgrid(np.arange(Y, dtype=np.float32), np.arange(X, dtype=np.float32), indexing="ij")
    yy = yy.reshape(-1) / np.float32(Y)
    xx = xx.reshape(-1) / np.float32(X)
    W = rng.normal(0.0, math.sqrt(1.0 / rank), size=(rank, d)).astype(np.float32)
    rho = np.float32(math.exp(-1.0 / tau))
    fresh_w = np.float32(math.sqrt(1.0 - float(rho) ** 2))
    out = np.empty((T, Y * X, d), dtype=np.float32)
    for t in range(T):
        fy = rng.integers(0, max_freq + 1, size=rank).astype(np.float32)
        fx = rng.integers(0, max_freq + 1, size=rank).astype(np.float32)
        ph = rng.uniform(0.0, 2.0 * math.pi, size=rank).astype(np.float32)
        U = np.cos(np.float32(2.0 * math.pi) * (np.outer(yy, fy) + np.outer(xx, fx)) + ph[None, :])
        cur = U @ W
        if t == 0:
            out[0] = cur
        else:
            np.multiply(out[t - 1], rho, out=out[t])
            out[t] += fresh_w * cur
    flat = out.reshape(T * Y * X, d)
    rms = math.sqrt(float(np.dot(flat.ravel(), flat.ravel())) / flat.size)
    if rms > 0:
        flat *= np.float32(1.0 / rms)
    return flat


def micro_heads(w: Workload) -> np.ndarray:
    """uint8 [H] flags of the heads that get Micro repair.

    Mode 2 (per-head percentile): the first round(frac * H) heads of a seeded
    permutation, drawn from an RNG stream separate from the tensors.  Other
    modes: every head.
    """
    flags = np.zeros(w.H, dtype=np.uint8)
    if w.micro_mode == 0:
        return flags
    if w.micro_mode != 2 or w.micro_head_frac >= 1.0:
        flags[:] = 1
        return flags
    rng = np.random.default_rng([w.seed, 1])
    perm = rng.permutation(w.H)
    n = round_half_up(w.micro_head_frac * w.H)
    flags[perm[:n]] = 1
    return flags


def make_qkv(w: Workload, heads: Optional[Tuple[int, int]] = None):
    """Draw Q, K, V for workload ``w``.

    Returns three float32 arrays of shape [B, H', N_pad, d] whose values are
    bfloat16-representable (H' = number of heads in ``heads`` = (h0, h1),
    default all).  Each head is drawn from its own seeded stream, so a head
    range is identical to the same heads cut from the full draw.
    """
    h0, h1 = heads if heads is not None else (0, w.H)
    N, Np, d = w.n_valid, w.n_pad, w.d
    out = [np.zeros((w.B, h1 - h0, Np, d), dtype=np.float32) for _ in range(3)]
    shared = None
    if w.generator == "tiny":
        shared = _tiny_field(np.random.default_rng([w.seed, 2]), w.grid, d)
    tail_rows = None
    if w.heavy_tail:
        trng = np.random.default_rng([w.seed, 3])
        tail_rows = np.sort(trng.choice(N, size=max(1, N // 100), replace=False))
    def one_head(b: int, h: int) -> None:
        rng = np.random.default_rng([w.seed, 0, b, h])
        if w.generator == "tiny":
            fqk = fv = shared
        else:
            fqk = _locality_field(rng, w.grid, d)
            fv = _locality_field(rng, w.grid, d)
        for idx, f in enumerate((fqk, fqk, fv)):
            x = rng.standard_normal(size=(N, d), dtype=np.float32)
            x += np.float32(w.field_scale) * f
            if tail_rows is not None and idx < 2:
                x[tail_rows] *= np.float32(4.0)
            out[idx][b, h - h0, :N] = round_to_bf16(x)

    jobs = [(b, h) for b in range(w.B) for h in range(h0, h1)]
    workers = min(len(jobs), max(1, (os.cpu_count() or 1)))
    if workers <= 1:
        for b, h in jobs:
            one_head(b, h)
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(lambda bh: one_head(*bh), jobs))
    return tuple(out)


def merge_sides(w: Workload, rounds: int, n_clusters: int, heads: Optional[Tuple[int, int]] = None) -> np.ndarray:
    """uint8 [B, H, rounds, n_clusters] random bipartition bits of the cluster
    merging rounds (one bit per query cluster and round; a group takes the
    bit of its lowest member), drawn from an RNG stream of their own."""
    h0, h1 = (0, w.H) if heads is None else heads
    out = np.zeros((w.B, h1 - h0, rounds, n_clusters), dtype=np.uint8)
    for b in range(w.B):
        for h in range(h0, h1):
            rng = np.random.default_rng([w.seed, 4, b, h])
            out[b, h - h0] = rng.integers(0, 2, size=(rounds, n_clusters), dtype=np.uint8)
    return out
