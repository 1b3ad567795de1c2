"""GPU parity of the forward over padded sequences of per-batch lengths
(``attn_fwd_varlen``): rows i < seqlens_q[b] of batch b must equal the fp64
oracle run on exactly that batch's first seqlens_q[b] query rows and first
seqlens_k[b] keys; padding rows are not written."""
import math

import numpy as np
import pytest
import torch

from scaled_dot_product_fa2_b200 import _lib
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


def run(sdpa, q, k, v, lq, lk, causal):
    qd, kd, vd = parity.to_dev(q, k, v)
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    return sdpa.attn_fwd_varlen(qd, kd, vd, sq, sk, causal=causal)


def check(o, lse, q, k, v, lq, lk, scale, causal, what):
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for b, (Lq, Lk) in enumerate(zip(lq, lk)):
        Lq = max(0, min(Lq, q.shape[2]))
        Lk = max(0, min(Lk, k.shape[2]))
        assert not np.any(o[b, :, Lq:]), f"{what}: padding rows of batch {b} were written"
        if Lq == 0:
            continue
        o_ref, lse_ref = parity.oracle_full(q[b:b + 1, :, :Lq], k[b:b + 1, :, :Lk], v[b:b + 1, :, :Lk], scale, causal)
        parity.compare(o[b:b + 1, :, :Lq], lse[b:b + 1, :, :Lq], o_ref, lse_ref, f"{what} batch {b}")


# ragged lengths: full, single row, empty, one past a tile; keys: full, none, ragged, exactly one tile
LQ, LK = [300, 1, 0, 129, 257], [517, 0, 200, 128, 517]


@pytest.mark.parametrize("causal,d,Hq,Hkv", [(NONE, 128, 2, 2), (TL, 128, 4, 2), (BR, 128, 2, 1), (BR, 64, 2, 2),
                                             (TL, 64, 2, 2)])
def test_fwd_varlen_matches_per_batch_oracle(sdpa, causal, d, Hq, Hkv):
    q, k, v = parity.seeded(len(LQ), Hq, Hkv, 300, 517, d, seed=800 + 10 * causal + d + Hq)
    o, lse = run(sdpa, q, k, v, LQ, LK, causal)
    sdpa.check_device_error()
    check(o, lse, q, k, v, LQ, LK, 1 / math.sqrt(d), causal, f"causal={causal} d={d} G={Hq // Hkv}")


def test_fwd_varlen_full_lengths_equal_fixed_length_forward(sdpa):
    B, Hq, Hkv, Sq, Sk = 2, 4, 2, 384, 640
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, 128, seed=81)
    for causal in (NONE, TL, BR):
        o1, l1 = run(sdpa, q, k, v, [Sq] * B, [Sk] * B, causal)
        qd, kd, vd = parity.to_dev(q, k, v)
        o2, l2 = sdpa.attn_fwd(qd, kd, vd, causal=causal)
        sdpa.check_device_error()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"causal={causal}"


def test_fwd_varlen_lengths_are_read_on_the_device(sdpa):
    B, Hq, Hkv, Sq, Sk = 3, 2, 2, 260, 300
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, 128, seed=82)
    qd, kd, vd = parity.to_dev(q, k, v)
    first, second = ([260, 5, 130], [300, 40, 129]), ([17, 260, 0], [1, 300, 300])
    sq = torch.tensor(first[0], dtype=torch.int32, device="cuda")
    sk = torch.tensor(first[1], dtype=torch.int32, device="cuda")
    o1, l1 = sdpa.attn_fwd_varlen(qd, kd, vd, sq, sk, causal=BR)
    o1, l1 = o1.clone(), l1.clone()
    sq.copy_(torch.tensor(second[0], dtype=torch.int32, device="cuda"))
    sk.copy_(torch.tensor(second[1], dtype=torch.int32, device="cuda"))
    o2, l2 = sdpa.attn_fwd_varlen(qd, kd, vd, sq, sk, causal=BR)
    sdpa.check_device_error()
    check(o1, l1, q, k, v, *first, 1 / math.sqrt(128), BR, "first lengths")
    check(o2, l2, q, k, v, *second, 1 / math.sqrt(128), BR, "second lengths")


def test_fwd_varlen_out_of_range_lengths_are_clamped_and_reported(sdpa):
    B, Hq, Hkv, Sq, Sk = 2, 2, 2, 130, 200
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, 128, seed=83)
    o, lse = run(sdpa, q, k, v, [Sq + 9, 60], [-4, Sk + 1], TL)
    with pytest.raises(_lib.AttnError) as err:
        sdpa.check_device_error()
    assert err.value.status == 13
    sdpa.check_device_error()
    check(o, lse, q, k, v, [Sq, 60], [0, Sk], 1 / math.sqrt(128), TL, "clamped")


def test_fwd_varlen_long_gqa_sampled_rows(sdpa):
    """GQA at long lengths (several 256-row units per batch, one much shorter
    batch), into NaN-filled outputs: every valid row must be written and every
    padding row left alone; one oracle row from every 128-row query tile of
    every head of both batches."""
    B, Hq, Hkv, S = 2, 32, 8, 4096
    lq, lk = [4096, 1500], [4096, 3000]
    q, k, v = parity.seeded(B, Hq, Hkv, S, S, 128, seed=84)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = parity.nan_outputs(qd, B, Hq, S)
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    sdpa.attn_fwd_varlen(qd, kd, vd, sq, sk, causal=BR, out=o, lse=lse)
    sdpa.check_device_error()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    scale = 1 / math.sqrt(128)
    for b in range(B):
        assert np.isfinite(o[b, :, :lq[b]]).all() and np.isfinite(lse[b, :, :lq[b]]).all(), f"batch {b} unwritten"
        assert np.isnan(o[b, :, lq[b]:]).all() and np.isnan(lse[b, :, lq[b]:]).all(), f"batch {b} padding written"
        rows = parity.tile_rows(1, Hq, lq[b], seed=5 + b)
        o_ref, lse_ref = parity.oracle_rows(q[b:b + 1, :, :lq[b]], k[b:b + 1, :, :lk[b]], v[b:b + 1, :, :lk[b]],
                                            scale, BR, rows)
        got_o = o[b, :, :lq[b]].reshape(-1, 128)[rows]
        got_l = lse[b, :, :lq[b]].reshape(-1)[rows]
        parity.compare(got_o, got_l, o_ref, lse_ref, f"batch {b}")
