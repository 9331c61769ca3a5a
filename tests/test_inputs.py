"""The seeded synthetic inputs: the recipe the workloads state, pinned.

The generators hold none of the method's arithmetic, but every parity test and
bench line stands on them, so the properties the workloads claim are checked
here against library routines and statistics rather than by re-running the
generator's own steps: bf16 rounding against torch's conversion, the
locality field's unit RMS and exp(-|dt|/3) frame correlation, the heavy tail
(1% of tokens x4 in Q and K, not in V), zero padding rows, head ranges equal
to the same heads of the full draw, and the Micro head count.
"""
import dataclasses
import math

import numpy as np
import torch

from video_inputs import WORKLOADS, Workload, make_qkv, micro_heads, round_to_bf16, sweep_points


def _small(heavy_tail=False, H=3, grid=(12, 8, 12), seed=7, generator="locality"):
    return Workload("small", 1, H, 32, grid, 128, 128, seed=seed, generator=generator, field_scale=0.8,
                    heavy_tail=heavy_tail, fixed_k=2)


def test_round_to_bf16_matches_torch_including_ties():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32) * np.float32(37.0),
        # exact ties between two bf16 neighbours (round to even either way)
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -126 * (1 + 2.0 ** -8)],
                 dtype=np.float32),
        np.array([0.0, -0.0, 1e-40, 3.4e38], dtype=np.float32),
    ])
    ours = round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_locality_field_unit_rms_and_frame_correlation():
    # Q and K of a head share one field; the field is what the noise adds to
    # both, so the cross-covariance of Q and K estimates its covariance
    w = _small(H=2, grid=(24, 16, 16), seed=11)
    q, k, _ = make_qkv(w)
    T, Y, X = w.grid
    s = np.float64(w.field_scale)
    for h in range(w.H):
        qh = q[0, h, :w.n_valid].astype(np.float64).reshape(T, Y * X, w.d)
        kh = k[0, h, :w.n_valid].astype(np.float64).reshape(T, Y * X, w.d)
        # E[q k] per element = field_scale^2 * field^2 (independent unit noise):
        # the field has unit mean square
        ms = float(np.mean(qh * kh)) / s ** 2
        assert abs(ms - 1.0) < 0.05, ms
        # frame correlation of the field, estimated across Q of frame t and K
        # of frame t + dt, decays as exp(-dt / 3)
        for dt in (1, 3, 6):
            c = float(np.mean(qh[:-dt] * kh[dt:])) / s ** 2
            assert abs(c - math.exp(-dt / 3.0)) < 0.12, (dt, c)


def test_heavy_tail_scales_one_percent_of_tokens_in_q_and_k_only():
    w = _small(heavy_tail=True, H=2, grid=(10, 16, 20))
    q, k, v = make_qkv(w)
    n = w.n_valid
    base = _small(heavy_tail=False, H=2, grid=(10, 16, 20))
    q0, k0, v0 = make_qkv(base)
    # the same seed and streams: scaled rows are exactly 4x (bf16 keeps x4 exact)
    for x, x0 in ((q, q0), (k, k0)):
        ratio_rows = np.all(x[0, :, :n] == np.float32(4.0) * x0[0, :, :n], axis=-1)
        same_rows = np.all(x[0, :, :n] == x0[0, :, :n], axis=-1)
        assert np.all(ratio_rows | same_rows)
        scaled = ratio_rows & ~same_rows
        # the same token rows in every head, 1% of the tokens
        assert np.all(scaled == scaled[0:1])
        assert scaled[0].sum() == n // 100
    assert np.array_equal(v, v0)
    assert np.array_equal(np.all(q[0, :, :n] != q0[0, :, :n], axis=-1), np.all(k[0, :, :n] != k0[0, :, :n], axis=-1))


def test_padding_rows_are_zero_and_values_are_bf16():
    w = dataclasses.replace(_small(), grid=(3, 7, 9))   # 189 tokens -> 256
    q, k, v = make_qkv(w)
    assert w.n_pad == 256
    for x in (q, k, v):
        assert np.all(x[:, :, w.n_valid:] == 0)
        assert np.array_equal(x, round_to_bf16(x))


def test_head_range_equals_the_same_heads_of_the_full_draw():
    w = _small(heavy_tail=True, H=4)
    full = make_qkv(w)
    part = make_qkv(w, heads=(1, 3))
    for a, b in zip(full, part):
        assert np.array_equal(a[:, 1:3], b)


def test_micro_heads_and_sweep_points():
    hun = WORKLOADS["hunyuan"]
    flags = micro_heads(hun)
    assert flags.dtype == np.uint8 and flags.sum() == round(0.25 * hun.H) == 6
    assert np.array_equal(flags, micro_heads(hun))           # seeded, reproducible
    assert micro_heads(WORKLOADS["tiny"]).sum() == WORKLOADS["tiny"].H   # top-k mode: every head
    assert micro_heads(WORKLOADS["wan13b"]).sum() == 0
    pts = sweep_points()
    assert [round(f, 2) for f, _ in pts] == [1.0, 0.5, 0.25, 0.15, 0.08] * 2
    assert [w.fixed_k for _, w in pts[:5]] == [929, 465, 232, 139, 74]
    assert {(w.bq, w.bk) for _, w in pts} == {(128, 128), (64, 128)}
