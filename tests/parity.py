"""Shared helpers for the GPU parity tests: run the CUDA path through the
C ABI and compare it with the fp64 oracle on the same seeded bf16 inputs.

Tolerances (bf16 output, N(0,1) inputs): max |err| <= 2e-2 and
mean |err| <= 2e-3 on O, |err| <= 1e-3 on LSE (absolute, natural log).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from scaled_dot_product_fa2_b200 import inputs

O_MAX_ERR = 2e-2
O_MEAN_ERR = 2e-3
LSE_ERR = 1e-3


def seeded(B, Hq, Hkv, Sq, Sk, d, seed):
    return inputs.make_qkv(B, Hq, Hkv, Sq, Sk, d, seed)


def to_dev(*ts):
    return [t.cuda() for t in ts]


def eff_scale(scale, d):
    return scale if scale != 0.0 else 1.0 / math.sqrt(d)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Element-wise comparison; fully masked rows must be exactly 0 / -inf."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert not np.isnan(o_gpu).any(), f"{what}: NaN in O"
    assert not np.isnan(lse_gpu).any(), f"{what}: NaN in LSE"
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= O_MAX_ERR, f"{what}: max |O err| {err.max():.3e}"
    assert err.mean() <= O_MEAN_ERR, f"{what}: mean |O err| {err.mean():.3e}"
    masked = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), masked), f"{what}: -inf pattern of LSE differs"
    if (~masked).any():
        lerr = np.abs(lse_gpu[~masked] - lse_ref[~masked])
        assert lerr.max() <= LSE_ERR, f"{what}: max |LSE err| {lerr.max():.3e}"
    return float(err.max()), float(err.mean())


def oracle_full(q, k, v, scale, causal):
    return oracle.attn_fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, causal)


def oracle_rows(q, k, v, scale, causal, rows):
    return oracle.attn_rows(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, causal, rows)


def nan_outputs(q, B, Hq, Sq):
    """Output buffers pre-filled with NaN: a row the kernel never writes stays
    NaN, so a skipped or mis-dealt work unit cannot pass as finite stale data."""
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, Sq), float("nan"), dtype=torch.float32, device=q.device)
    return o, lse


def tile_rows(B, Hq, Sq, seed=0, tile=128):
    """Flattened rows: one seeded random row inside every ``tile``-row query
    tile of every (batch, head), plus each head's first and last row.  Each
    work unit of the forward (a batch, a head, a pair of 128-row query tiles)
    then has rows of both its tiles in the sample."""
    rng = np.random.default_rng(seed)
    n_t = (Sq + tile - 1) // tile
    bh = np.repeat(np.arange(B * Hq, dtype=np.int64), n_t)
    t = np.tile(np.arange(n_t, dtype=np.int64), B * Hq)
    size = np.minimum(tile, Sq - t * tile)
    i = t * tile + (rng.random(bh.shape[0]) * size).astype(np.int64)
    edges = np.concatenate([np.arange(B * Hq, dtype=np.int64) * Sq, np.arange(B * Hq, dtype=np.int64) * Sq + Sq - 1])
    return np.unique(np.concatenate([bh * Sq + i, edges]))


def sample_rows(B, Hq, Sq, n_random=96, seed=0):
    """Flattened (b*Hq + h)*Sq + i rows: tile edges, the ragged end, random rows."""
    rng = np.random.default_rng(seed)
    picks = set()
    heads = sorted({0, B * Hq - 1, int(rng.integers(0, B * Hq))})
    for bh in heads:
        for i in (0, 1, 127, 128, 255, 256, Sq // 2, Sq - 2, Sq - 1):
            if 0 <= i < Sq:
                picks.add(bh * Sq + i)
    for r in rng.integers(0, B * Hq * Sq, size=n_random):
        picks.add(int(r))
    return np.array(sorted(picks), dtype=np.int64)
