"""GPU parity with an additive attention bias (the decode page's attention
bias, applied with the mask; leading dims broadcast over batch and heads):
forward and split-KV decode against the fp64 oracle with the same bf16 bias."""
import math

import numpy as np
import pytest
import torch

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


def make_bias(dims, Sq, Sk, seed, masked=True):
    """bf16 bias N(0, 2^2) with, optionally, a few -inf entries (masked keys)."""
    g = torch.Generator().manual_seed(seed)
    bias = (torch.randn((*dims, Sq, Sk), generator=g) * 2.0)
    if masked:
        drop = torch.rand((*dims, Sq, Sk), generator=g) < 0.05
        bias[drop] = -math.inf
    return bias.bfloat16()


def oracle(q, k, v, bias, causal, d):
    return parity.oracle_full(q, k, v, 1 / math.sqrt(d), causal) if bias is None else tuple(
        __import__("oracle").attn_fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                      1 / math.sqrt(d), causal, bias=bias.double().numpy()))


@pytest.mark.parametrize("dims", ["11", "B1", "1H", "BH"])
@pytest.mark.parametrize("causal", [NONE, TL, BR])
def test_forward_bias_matches_oracle(sdpa, dims, causal):
    B, Hq, Hkv, Sq, Sk, d = 2, 4, 2, 300, 520, 128
    shape = (B if dims[0] == "B" else 1, Hq if dims[1] == "H" else 1)
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=900 + causal)
    bias = make_bias(shape, Sq, Sk, seed=901 + causal)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_fwd(qd, kd, vd, causal=causal, bias=bias.cuda())
    sdpa.check_device_error()
    o_ref, lse_ref = oracle(q, k, v, bias, causal, d)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"fwd bias {dims} causal={causal}")


def test_forward_bias_d64_gqa_and_zero_bias_equals_no_bias(sdpa):
    B, Hq, Hkv, Sq, Sk, d = 1, 8, 2, 257, 384, 64
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=910)
    bias = make_bias((1, Hq), Sq, Sk, seed=911)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = sdpa.attn_fwd(qd, kd, vd, causal=BR, bias=bias.cuda())
    sdpa.check_device_error()
    o_ref, lse_ref = oracle(q, k, v, bias, BR, d)
    parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fwd bias d64")
    zero = torch.zeros((1, 1, Sq, Sk), dtype=torch.bfloat16, device="cuda")
    o1, l1 = sdpa.attn_fwd(qd, kd, vd, causal=TL, bias=zero)
    o2, l2 = sdpa.attn_fwd(qd, kd, vd, causal=TL)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [NONE, TL])
def test_forward_bias_many_units_sampled_rows(sdpa, causal):
    """More work units than SMs (2 x 16 heads x 8 units of 256 rows), so every
    CTA takes several units and the bias tiles stream through their staging
    buffer across unit boundaries (and, causal, past the shorter tile's last
    step); outputs NaN-prefilled; one oracle row from every 128-row tile."""
    import oracle as oracle_mod
    B, Hq, Hkv, S, d = 2, 16, 16, 2048, 128
    q, k, v = parity.seeded(B, Hq, Hkv, S, S, d, seed=930 + causal)
    bias = make_bias((1, Hq), S, S, seed=931 + causal)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = parity.nan_outputs(qd, B, Hq, S)
    sdpa.attn_fwd(qd, kd, vd, causal=causal, bias=bias.cuda(), out=o, lse=lse)
    sdpa.check_device_error()
    # written rows are finite (a row whose every key is masked has O = 0, LSE = -inf)
    assert not torch.isnan(o).any() and not torch.isnan(lse).any(), "a row was never written"
    rows = parity.tile_rows(B, Hq, S, seed=932 + causal)
    o_ref, lse_ref = oracle_mod.attn_rows(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                          1 / math.sqrt(d), causal, rows, bias=bias.double().numpy())
    got_o = o.float().cpu().numpy().reshape(-1, d)[rows]
    got_l = lse.cpu().numpy().reshape(-1)[rows]
    parity.compare(got_o, got_l, o_ref, lse_ref, f"fwd bias many units causal={causal}")


@pytest.mark.parametrize("dims", ["11", "BH"])
@pytest.mark.parametrize("Sq,causal", [(1, BR), (4, BR), (3, NONE)])
def test_decode_bias_matches_oracle(sdpa, dims, Sq, causal):
    B, Hq, Hkv, Sk, d = 2, 8, 2, 777, 128  # odd Sk: the decode reads bias element by element
    shape = (B if dims[0] == "B" else 1, Hq if dims[1] == "H" else 1)
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=920 + Sq)
    bias = make_bias(shape, Sq, Sk, seed=921 + Sq)
    qd, kd, vd = parity.to_dev(q, k, v)
    for splits in (0, 1, 5):
        o, lse = sdpa.attn_decode_splitkv(qd, kd, vd, causal=causal, num_splits=splits, bias=bias.cuda())
        sdpa.check_device_error()
        o_ref, lse_ref = oracle(q, k, v, bias, causal, d)
        parity.compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref,
                       f"decode bias {dims} Sq={Sq} splits={splits}")


def test_decode_bias_with_per_batch_lengths(sdpa):
    """Bias and device-side lengths together: each batch against the oracle on
    its prefix of keys and the matching columns of the bias."""
    B, Hq, Hkv, Sq, cap, d = 3, 4, 2, 2, 600, 128
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, cap, d, seed=930)
    bias = make_bias((B, Hq), Sq, cap, seed=931)
    lens = [600, 77, 1]
    qd, kd, vd = parity.to_dev(q, k, v)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = sdpa.attn_decode_splitkv(qd, kd, vd, causal=BR, bias=bias.cuda(), seqlens_k=sl)
    sdpa.check_device_error()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    import oracle as orc
    for b, L in enumerate(lens):
        o_ref, lse_ref = orc.attn_fwd(q[b:b + 1].double().numpy(), k[b:b + 1, :, :L].double().numpy(),
                                      v[b:b + 1, :, :L].double().numpy(), 1 / math.sqrt(d), BR,
                                      bias=bias[b:b + 1, :, :, :L].double().numpy())
        parity.compare(o[b:b + 1], lse[b:b + 1], o_ref, lse_ref, f"batch {b}")


@pytest.mark.parametrize("causal", [TL, BR])
def test_forward_bias_with_per_batch_lengths(sdpa, causal):
    """Bias and per-batch lengths together (attn_fwd_ex with both extras):
    the run-time unit hand-out and the bias loader walk the same units; each
    batch's valid rows equal the oracle on its own rows, keys and bias block."""
    import ctypes
    from scaled_dot_product_fa2_b200 import _lib
    B, Hq, Hkv, S, d = 3, 4, 2, 600, 128
    lq, lk = [600, 130, 257], [600, 416, 257]
    q, k, v = parity.seeded(B, Hq, Hkv, S, S, d, seed=940 + causal)
    bias = make_bias((1, Hq), S, S, seed=941 + causal)
    qd, kd, vd = parity.to_dev(q, k, v)
    o, lse = parity.nan_outputs(qd, B, Hq, S)
    bd = bias.cuda()
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    ex = _lib.Extras()
    ex.seqlens_q, ex.seqlens_k, ex.bias = sq.data_ptr(), sk.data_ptr(), bd.data_ptr()
    ex.bias_b, ex.bias_h, ex.layout = 1, Hq, 0
    st = _lib.get().attn_fwd_ex(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                                S, S, d, 0.0, causal, ctypes.byref(ex), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    sdpa.check_device_error()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for b in range(B):
        assert np.isnan(o[b, :, lq[b]:]).all(), f"batch {b}: padding rows written"
        o_ref, lse_ref = oracle(q[b:b + 1, :, :lq[b]], k[b:b + 1, :, :lk[b]], v[b:b + 1, :, :lk[b]],
                                bias[:, :, :lq[b], :lk[b]].contiguous(), causal, d)
        parity.compare(o[b:b + 1, :, :lq[b]], lse[b:b + 1, :, :lq[b]], o_ref, lse_ref, f"bias varlen batch {b}")
