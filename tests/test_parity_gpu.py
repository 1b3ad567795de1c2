"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element in full (several 128-row tiles,
ragged tails, every causal mode, GQA, d = 64 and 128, edge cases).  The
full-size workloads run in the launch configuration the benchmark uses, into
NaN-filled outputs (every row must be written): each is compared on one
oracle row from every 128-row query tile, and two whole workloads (causal
seq 2048, non-causal seq 4096) element by element.
"""
import math

import numpy as np
import pytest
import torch

from scaled_dot_product_fa2_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu

NONE, TL, BR = 0, 1, 2


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scaled_dot_product_fa2_b200 import build
    build.build()
    import scaled_dot_product_fa2_b200 as m
    return m


def run_fwd(sdpa, B, Hq, Hkv, Sq, Sk, d, causal, seed, scale=0.0):
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    sdpa.check_device_error()
    return (q, k, v), o.float().cpu().numpy(), lse.cpu().numpy()


# ------------------------------------------------------------- small, full compare

SMALL = [
    # B, Hq, Hkv, Sq, Sk, d, causal
    (1, 2, 2, 128, 128, 64, TL),       # the tiny workload's shape
    (2, 2, 2, 300, 300, 128, NONE),    # ragged tail, 2 CTA units
    (2, 2, 2, 300, 300, 128, TL),
    (1, 3, 3, 517, 517, 128, TL),      # odd heads, 3 units, ragged
    (1, 2, 2, 200, 517, 128, BR),      # queries at the end of longer keys
    (1, 2, 2, 200, 517, 128, TL),
    (1, 2, 2, 200, 517, 128, NONE),
    (1, 2, 2, 517, 200, 128, BR),      # Sq > Sk: first rows fully masked
    (1, 2, 2, 517, 200, 128, TL),
    (1, 8, 2, 384, 384, 128, TL),      # GQA group 4
    (2, 4, 1, 256, 640, 128, NONE),    # GQA group 4, Sk multiple of 128
    (1, 2, 2, 300, 300, 64, NONE),     # d = 64
    (1, 4, 2, 333, 333, 64, TL),
    (1, 2, 2, 100, 700, 64, BR),
    (1, 2, 2, 1, 1, 128, NONE),        # single row, single key
    (1, 2, 2, 1, 1000, 128, BR),       # one query at the end of 1000 keys
    (3, 2, 2, 7, 129, 128, NONE),      # ragged both ways, tiny
    (1, 1, 1, 1024, 1024, 128, TL),    # 4 units, exercises LPT ordering
    (4, 40, 8, 520, 520, 128, TL),     # 480 units > 148 CTAs, one CTA per unit taken over at run time, GQA group 5
    (4, 40, 8, 520, 520, 128, NONE),   # 480 units over the 148-CTA persistent grid: several dealing rounds
    (3, 32, 32, 300, 700, 64, BR),     # 192 units > 148 CTAs at d = 64 (8-slot ring)
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}_H{}x{}_Sq{}_Sk{}_d{}_c{}".format(*s))
def test_prefill_small_full_compare(sdpa, shape):
    B, Hq, Hkv, Sq, Sk, d, causal = shape
    (q, k, v), o, lse = run_fwd(sdpa, B, Hq, Hkv, Sq, Sk, d, causal, seed=hash(shape) % 10000)
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1.0 / math.sqrt(d), causal)
    parity.compare(o, lse, o_ref, lse_ref, what=str(shape))


def test_tiny_workload_fp32_inputs_rounded(sdpa):
    """The tiny causal workload: fp32 N(0,1) inputs, rounded once to bf16 for both sides."""
    w = inputs.TINY
    q32, k32, v32 = inputs.workload_inputs(w, dtype=torch.float32)
    q, k, v = q32.bfloat16(), k32.bfloat16(), v32.bfloat16()
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale)
    sdpa.check_device_error()
    o_ref, lse_ref = parity.oracle_full(q, k, v, w.scale, w.causal)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "tiny")
    # row 0 of a causal mask is exactly v[0] (up to bf16 output rounding)
    np.testing.assert_allclose(o.float().cpu()[:, :, 0].numpy(), v.float()[:, :, 0].numpy(), atol=1e-2)


def test_custom_scale(sdpa):
    (q, k, v), o, lse = run_fwd(sdpa, 1, 2, 2, 260, 260, 128, TL, seed=7, scale=0.05)
    o_ref, lse_ref = parity.oracle_full(q, k, v, 0.05, TL)
    parity.compare(o, lse, o_ref, lse_ref, "scale=0.05")


def test_no_keys_gives_zero_and_neg_inf(sdpa):
    q = torch.randn(1, 2, 5, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")
    o, lse = sdpa.attn_fwd(q, k, k.clone(), causal=NONE)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_lse_optional(sdpa):
    q, k, v = parity.to_dev(*parity.seeded(1, 2, 2, 130, 130, 128, 11))
    o1, lse = sdpa.attn_fwd(q, k, v, causal=TL)
    o2, none = sdpa.attn_fwd(q, k, v, causal=TL, return_lse=False)
    torch.cuda.synchronize()
    assert none is None and torch.equal(o1, o2)


def test_deterministic(sdpa):
    q, k, v = parity.to_dev(*parity.seeded(2, 4, 2, 700, 700, 128, 12))
    a = sdpa.attn_fwd(q, k, v, causal=TL)
    b = sdpa.attn_fwd(q, k, v, causal=TL)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_large_magnitude_inputs_stay_finite(sdpa):
    """Scores spanning hundreds of units force the rare O-rescale path."""
    q, k, v = parity.seeded(1, 2, 2, 384, 384, 128, 13)
    q = (q.float() * 4).bfloat16()
    k = (k.float() * 4).bfloat16()
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_fwd(qd, kd, vd, causal=TL)
    sdpa.check_device_error()
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(128), TL)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "large scores")


# ------------------------------------------------------------- full-size workloads

FULL = inputs.PREFILL_NONCAUSAL + inputs.PREFILL_CAUSAL + [inputs.GQA_LONG]


def run_full_size(sdpa, w):
    """The workload in the benchmark's launch configuration, into NaN-filled outputs."""
    q, k, v = inputs.workload_inputs(w)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = parity.nan_outputs(qd, w.B, w.Hq, w.Sq)
    sdpa.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse)
    sdpa.check_device_error()
    # every row of every work unit was written (the buffers started as NaN)
    assert torch.isfinite(o).all(), f"{w.name}: rows of O left unwritten"
    assert torch.isfinite(lse).all(), f"{w.name}: LSE entries left unwritten"
    return (q, k, v), o, lse


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_prefill_full_size_every_tile_sampled(sdpa, w):
    """One oracle row inside every 128-row query tile of every head, so every
    work unit is checked against the oracle, not only a random handful: all
    rounds of the persistent grid's snake dealing (non-causal) and every unit
    taken over at run time (causal, GQA)."""
    (q, k, v), o, lse = run_full_size(sdpa, w)
    rows = parity.tile_rows(w.B, w.Hq, w.Sq, seed=w.seed)
    o_ref, lse_ref = parity.oracle_rows(q, k, v, w.eff_scale, w.causal, rows)
    idx = torch.from_numpy(rows).cuda()
    o_g = o.reshape(-1, w.d)[idx].float().cpu().numpy()
    l_g = lse.reshape(-1)[idx].cpu().numpy()
    parity.compare(o_g, l_g, o_ref, lse_ref, w.name)


WHOLE = [inputs.BY_NAME["prefill_causal_s2048"], inputs.BY_NAME["prefill_noncausal_s4096"]]


@pytest.mark.parametrize("w", WHOLE, ids=lambda w: w.name)
def test_prefill_whole_workload_element_by_element(sdpa, w):
    """Every element of a whole benchmark workload against the oracle: causal
    seq 2048 (1024 work units, one CTA per unit, units taken over at run time
    by running CTAs) and non-causal seq 4096 (512 units over the 148-CTA
    persistent grid: the multi-round snake dealing and the ring and barrier
    phases that run on across units), checked on every row."""
    (q, k, v), o, lse = run_full_size(sdpa, w)
    o_ref, lse_ref = parity.oracle_full(q, k, v, w.eff_scale, w.causal)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, w.name)


# ------------------------------------------------------------- decode

def run_decode(sdpa, B, Hq, Hkv, Sq, Sk, d, causal, seed, num_splits=0):
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_decode_splitkv(qd, kd, vd, causal=causal, num_splits=num_splits)
    sdpa.check_device_error()
    return (q, k, v), o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("w", inputs.DECODE, ids=lambda w: w.name)
def test_decode_workload_full_compare(sdpa, w):
    q, k, v = inputs.workload_inputs(w)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_decode_splitkv(qd, kd, vd, causal=w.causal)
    sdpa.check_device_error()
    o_ref, lse_ref = parity.oracle_full(q, k, v, w.eff_scale, w.causal)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, w.name)


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 16, 128, 1000])
def test_decode_split_sweep_equals_unsplit_oracle(sdpa, splits):
    (q, k, v), o, lse = run_decode(sdpa, 2, 8, 2, 4, 8192, 128, BR, seed=20 + splits, num_splits=splits)
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(128), BR)
    parity.compare(o, lse, o_ref, lse_ref, f"splits={splits}")


DECODE_SMALL = [
    (1, 4, 1, 1, 1000, 128, BR),     # ragged Sk
    (2, 8, 2, 3, 777, 128, BR),
    (1, 32, 2, 4, 300, 128, BR),     # G*Sq = 64 rows: 4 row groups
    (2, 4, 4, 2, 513, 64, BR),       # d = 64, G = 1
    (1, 4, 2, 5, 250, 128, NONE),
    (1, 4, 2, 5, 250, 128, TL),
    (1, 2, 1, 9, 6, 128, BR),        # Sq > Sk: fully masked rows
    (1, 2, 2, 1, 1, 128, BR),
]


@pytest.mark.parametrize("shape", DECODE_SMALL, ids=lambda s: "B{}_H{}x{}_Sq{}_Sk{}_d{}_c{}".format(*s))
def test_decode_small_full_compare(sdpa, shape):
    B, Hq, Hkv, Sq, Sk, d, causal = shape
    for splits in (0, 1, 3):
        (q, k, v), o, lse = run_decode(sdpa, B, Hq, Hkv, Sq, Sk, d, causal, seed=hash(shape) % 997,
                                       num_splits=splits)
        o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(d), causal)
        parity.compare(o, lse, o_ref, lse_ref, f"{shape} splits={splits}")


def test_decode_matches_prefill_kernel(sdpa):
    q, k, v = parity.to_dev(*parity.seeded(2, 8, 2, 4, 2048, 128, 30))
    o1, l1 = sdpa.attn_decode_splitkv(q, k, v, causal=BR)
    o2, l2 = sdpa.attn_fwd(q, k, v, causal=BR)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3
