"""GPU parity of the token-major [B, S, H, d] layout (ATTN_LAYOUT_BSHD): the
forward with q, k, v, o in that layout and the decode with q, o in it must
equal the fp64 oracle (fed the same values in [B, H, S, d]) and, bit for bit,
the default layout's result."""
import math

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


def bshd(t):
    return t.transpose(1, 2).contiguous()


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,d,causal", [
    (2, 4, 2, 300, 517, 128, NONE),
    (2, 4, 2, 300, 300, 128, TL),
    (1, 8, 2, 200, 517, 128, BR),
    (1, 2, 2, 333, 333, 64, TL),
    (3, 2, 1, 7, 129, 128, NONE),
])
def test_forward_bshd_matches_oracle_and_default_layout(sdpa, B, Hq, Hkv, Sq, Sk, d, causal):
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=1000 + Sq + causal)
    qd, kd, vd = parity.to_dev(q, k, v)
    o1, l1 = sdpa.attn_fwd(bshd(qd), bshd(kd), bshd(vd), causal=causal, layout=sdpa.LAYOUT_BSHD)
    o2, l2 = sdpa.attn_fwd(qd, kd, vd, causal=causal)
    sdpa.check_device_error()
    assert tuple(o1.shape) == (B, Sq, Hq, d)
    o1 = o1.transpose(1, 2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(d), causal)
    parity.compare(o1.float().cpu().numpy(), l1.cpu().numpy(), o_ref, lse_ref, "bshd forward")


def test_forward_bshd_with_bias(sdpa):
    B, Hq, Hkv, Sq, Sk, d = 2, 4, 2, 256, 384, 128
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=1010)
    bias = (torch.randn((1, Hq, Sq, Sk), generator=torch.Generator().manual_seed(1011)) * 2).bfloat16()
    qd, kd, vd = parity.to_dev(q, k, v)
    o1, l1 = sdpa.attn_fwd(bshd(qd), bshd(kd), bshd(vd), causal=BR, bias=bias.cuda(), layout=sdpa.LAYOUT_BSHD)
    o2, l2 = sdpa.attn_fwd(qd, kd, vd, causal=BR, bias=bias.cuda())
    sdpa.check_device_error()
    assert torch.equal(o1.transpose(1, 2), o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("Sq", [1, 4])
def test_decode_bshd_query_matches_default_layout(sdpa, Sq):
    B, Hq, Hkv, Sk, d = 3, 8, 2, 1000, 128
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=1020 + Sq)
    qd, kd, vd = parity.to_dev(q, k, v)
    for splits in (0, 3):
        o1, l1 = sdpa.attn_decode_splitkv(bshd(qd), kd, vd, causal=BR, num_splits=splits,
                                          layout=sdpa.LAYOUT_BSHD)
        o2, l2 = sdpa.attn_decode_splitkv(qd, kd, vd, causal=BR, num_splits=splits)
        sdpa.check_device_error()
        assert tuple(o1.shape) == (B, Sq, Hq, d)
        assert torch.equal(o1.transpose(1, 2), o2) and torch.equal(l1, l2)
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(d), BR)
    parity.compare(o1.transpose(1, 2).float().cpu().numpy(), l1.cpu().numpy(), o_ref, lse_ref, "bshd decode")


@pytest.mark.parametrize("d,causal,layout", [(128, TL, 0), (64, NONE, 0), (128, BR, 1)])
def test_forward_output_aligned_to_16_bytes_only(sdpa, d, causal, layout):
    """An output buffer 16 bytes past a 32-byte boundary takes the epilogue's
    16-byte store path; it must write the same bits as a 32-byte aligned one."""
    from scaled_dot_product_fa2_b200 import ops
    B, Hq, Hkv, Sq, Sk = 2, 4, 2, 300, 517
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=1300 + d + causal)
    qd, kd, vd = parity.to_dev(q, k, v)
    lay = ops.LAYOUT_BSHD if layout else ops.LAYOUT_BHSD
    if layout:
        qd, kd, vd = bshd(qd), bshd(kd), bshd(vd)
    o_ref, l_ref = sdpa.attn_fwd(qd, kd, vd, causal=causal, layout=lay)
    flat = torch.full((qd.numel() + 64,), float("nan"), dtype=torch.bfloat16, device="cuda")
    start = (32 - flat.data_ptr() % 32) // 2 + 8  # 16 bytes past a 32-byte boundary
    o_off = flat[start:start + qd.numel()].view(qd.shape)
    assert o_off.data_ptr() % 32 == 16
    o2, l2 = sdpa.attn_fwd(qd, kd, vd, causal=causal, layout=lay, out=o_off)
    sdpa.check_device_error()
    assert torch.equal(o2, o_ref) and torch.equal(l2, l_ref)
    assert torch.isnan(flat[:start]).all() and torch.isnan(flat[start + qd.numel():]).all()
