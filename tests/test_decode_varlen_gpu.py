"""GPU parity of the split-KV decode over caches with per-batch valid lengths
(``attn_decode_splitkv_varlen``): for every batch b the result must equal
attention over the first seqlens_k[b] keys of its cache, computed by the fp64
oracle on exactly that prefix; the lengths live in device memory and are read
by the kernels only."""
import math

import numpy as np
import pytest
import torch

from scaled_dot_product_fa2_b200 import _lib, inputs
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


def per_batch_oracle(q, k, v, lens, scale, causal):
    """Oracle on each batch's valid prefix of the cache, stacked."""
    outs, lses = [], []
    for b, L in enumerate(lens):
        L = max(0, min(int(L), k.shape[2]))
        o, l = parity.oracle_full(q[b:b + 1], k[b:b + 1, :, :L], v[b:b + 1, :, :L], scale, causal)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses)


def run_varlen(sdpa, q, k, v, lens, causal, num_splits=0):
    qd, kd, vd = parity.to_dev(q, k, v)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = sdpa.attn_decode_splitkv_varlen(qd, kd, vd, sl, causal=causal, num_splits=num_splits)
    return o, lse


# capacity 1000 (not a multiple of 64); lengths: empty, one key, fewer keys than
# query rows, a ragged middle, one short of capacity, exactly the capacity
LENS = [0, 1, 3, 517, 999, 1000]


@pytest.mark.parametrize("Sq,causal,d", [(1, BR, 128), (4, BR, 128), (4, NONE, 128), (3, TL, 128), (4, BR, 64)])
def test_varlen_matches_per_batch_oracle(sdpa, Sq, causal, d):
    B, Hq, Hkv, cap = len(LENS), 8, 2, 1000
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, d, seed=700 + Sq + 10 * causal + d)
    for splits in (0, 1, 5):
        o, lse = run_varlen(sdpa, q, k, v, LENS, causal, num_splits=splits)
        sdpa.check_device_error()
        o_ref, lse_ref = per_batch_oracle(q, k, v, LENS, 1 / math.sqrt(d), causal)
        parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref,
                       f"Sq={Sq} causal={causal} d={d} splits={splits}")


def test_varlen_full_lengths_match_fixed_length_decode(sdpa):
    B, Hq, Hkv, Sq, cap = 3, 8, 2, 4, 2048
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, 128, seed=71)
    o1, l1 = run_varlen(sdpa, q, k, v, [cap] * B, BR)
    qd, kd, vd = parity.to_dev(q, k, v)
    o2, l2 = sdpa.attn_decode_splitkv(qd, kd, vd, causal=BR)
    sdpa.check_device_error()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(128), BR)
    parity.compare(o1.float().cpu().numpy(), l1.cpu().numpy(), o_ref, lse_ref, "full lengths")


def test_varlen_lengths_are_read_on_the_device(sdpa):
    """Lengths rewritten by device work on the stream between two calls (no host
    synchronisation) take effect: nothing about them is cached on the host."""
    B, Hq, Hkv, Sq, cap = 4, 8, 2, 2, 640
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, 128, seed=72)
    qd, kd, vd = parity.to_dev(q, k, v)
    first, second = [640, 100, 5, 300], [64, 639, 200, 0]
    sl = torch.tensor(first, dtype=torch.int32, device="cuda")
    staged = torch.tensor(second, dtype=torch.int32, device="cuda")
    o1, l1 = sdpa.attn_decode_splitkv_varlen(qd, kd, vd, sl, causal=BR)
    o1, l1 = o1.clone(), l1.clone()
    sl.copy_(staged)  # same stream, after the first call
    o2, l2 = sdpa.attn_decode_splitkv_varlen(qd, kd, vd, sl, causal=BR)
    sdpa.check_device_error()
    for o, l, lens in ((o1, l1, first), (o2, l2, second)):
        o_ref, lse_ref = per_batch_oracle(q, k, v, lens, 1 / math.sqrt(128), BR)
        parity.compare(o.float().cpu().numpy(), l.cpu().numpy(), o_ref, lse_ref, f"lens={lens}")


def test_varlen_out_of_range_lengths_are_clamped_and_reported(sdpa):
    B, Hq, Hkv, Sq, cap = 2, 4, 2, 1, 300
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, 128, seed=73)
    o, lse = run_varlen(sdpa, q, k, v, [cap + 7, -3], BR)
    with pytest.raises(_lib.AttnError) as err:
        sdpa.check_device_error()
    assert err.value.status == 13
    sdpa.check_device_error()  # the error word was cleared
    o_ref, lse_ref = per_batch_oracle(q, k, v, [cap, 0], 1 / math.sqrt(128), BR)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "clamped")


@pytest.mark.parametrize("w", inputs.DECODE, ids=lambda w: w.name)
def test_varlen_decode_workload_sampled_rows(sdpa, w):
    """The decode workload's shapes with seeded lengths in [1, capacity]; every
    row of every batch is checked against the oracle on its prefix."""
    q, k, v = inputs.workload_inputs(w)
    lens = inputs.decode_lengths(w)
    o, lse = run_varlen(sdpa, q, k, v, lens, w.causal)
    sdpa.check_device_error()
    o_ref, lse_ref = per_batch_oracle(q, k, v, lens, w.eff_scale, w.causal)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, w.name + " varlen")



SKEWED = [
    # lengths, Hq, Hkv, Sq, capacity
    ([8192] + [0] * 7, 32, 8, 4, 8192),                       # one full batch, the rest empty
    ([5, 4000, 0, 8191, 64, 65, 1, 3000] * 5, 8, 2, 1, 8192),  # 40 batches of every kind of length
    ([300, 1, 299], 64, 2, 1, 300),                           # 32 query rows per kv head: two row groups
    ([2] * 200, 4, 4, 1, 64),                                 # 800 (batch, kv head) pairs, more than one wave
    ([5, 2000, 0, 2047] * 32, 4, 1, 1, 2048),                 # 128 batches: the largest dealt batch count
    ([7, 1000, 0, 513] * 40, 4, 1, 1, 1000),                  # 160 batches: tiles spread evenly per batch
]


@pytest.mark.parametrize("lens,Hq,Hkv,Sq,cap", SKEWED,
                         ids=["one_full", "b40", "two_row_groups", "many_pairs", "b128", "b160"])
def test_varlen_skewed_length_mixes(sdpa, lens, Hq, Hkv, Sq, cap):
    """Extreme mixes of per-batch lengths against the per-batch oracle, with the
    automatic split count and with fixed ones (the slots of a kv head are dealt
    to batches by their lengths, so the split count changes every batch's share)."""
    B = len(lens)
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, 128, seed=740 + B + Hq)
    o_ref, lse_ref = per_batch_oracle(q, k, v, lens, 1 / math.sqrt(128), BR)
    for splits in (0, 3, 16):
        o, lse = run_varlen(sdpa, q, k, v, lens, BR, num_splits=splits)
        sdpa.check_device_error()
        parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref,
                       f"lens {lens[:4]} splits={splits}")


def test_workspace_contents_do_not_matter(sdpa):
    """Whatever the caller's workspace holds before a call (never written,
    another call's leftovers) gives the same bits: the per-batch slot ranges and
    the partials are written by the call before anything reads them."""
    B, Hq, Hkv, Sq, cap = 6, 8, 2, 4, 1000
    lens = [1000, 3, 0, 517, 64, 999]
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, 128, seed=75)
    qd, kd, vd = parity.to_dev(q, k, v)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = sdpa.decode_workspace(qd, kd)
    results = []
    for fill in (0x00, 0xFF, 0x5A, None, None):
        if fill is not None:
            ws.fill_(fill)
        o, lse = sdpa.attn_decode_splitkv_varlen(qd, kd, vd, sl, causal=BR, workspace=ws)
        results.append((o.clone(), lse.clone()))
    sdpa.check_device_error()
    for o, lse in results[1:]:
        assert torch.equal(o, results[0][0]) and torch.equal(lse, results[0][1])
    o_ref, lse_ref = per_batch_oracle(q, k, v, lens, 1 / math.sqrt(128), BR)
    parity.compare(results[0][0].float().cpu().numpy(), results[0][1].cpu().numpy(), o_ref, lse_ref, "ws")
