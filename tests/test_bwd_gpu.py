"""GPU parity of the backward pass (``attn_bwd``) against the fp64 oracle
``oracle.attn_bwd`` on the same seeded bf16 q, k, v and dout.

The GPU side runs the library's own forward first (o, lse) and feeds them to
the backward, as a training step does.  Bar (relative to the largest
reference gradient G = max(max |ref|, 1e-3) of each tensor, the forward's
absolute bar scaled to the gradient's size): max |gpu - ref| <= 2e-2 G and
mean |gpu - ref| <= 2e-3 G.  The GPU rounds o, P and dS to bf16 (2^-9
relative each) before they enter fp32 sums, and the output to bf16.  The
floor 1e-3 on G covers gradients that are exactly zero (one key: dq = 0),
where the GPU's dP - D is a difference of two fp32 sums that round apart
(~1e-7).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from scaled_dot_product_fa2_b200 import inputs

pytestmark = pytest.mark.gpu

NONE, TL, BR = 0, 1, 2
MAX_REL = 2e-2
MEAN_REL = 2e-3


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scaled_dot_product_fa2_b200 import build
    build.build()
    import scaled_dot_product_fa2_b200 as m
    return m


def seeded_dout(B, Hq, Sq, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((B, Hq, Sq, d), generator=g).bfloat16()


def compare(gpu, ref, what):
    gpu = gpu.double().cpu().numpy()
    assert not np.isnan(gpu).any(), f"{what}: NaN"
    G = max(np.abs(ref).max(), 1e-3)
    err = np.abs(gpu - ref)
    assert err.max() <= MAX_REL * G, f"{what}: max err {err.max():.3e} > {MAX_REL} x {G:.3e}"
    assert err.mean() <= MEAN_REL * G, f"{what}: mean err {err.mean():.3e} > {MEAN_REL} x {G:.3e}"
    print(f"{what}: max {err.max() / G:.2e} mean {err.mean() / G:.2e} of G={G:.3e}")
    return err.max() / G, err.mean() / G


def run_case(sdpa, B, Hq, Hkv, Sq, Sk, d, causal, seed, scale=0.0):
    q, k, v = inputs.make_qkv(B, Hq, Hkv, Sq, Sk, d, seed)
    dout = seeded_dout(B, Hq, Sq, d, seed + 1)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = sdpa.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = sdpa.attn_bwd(qd, kd, vd, o, lse, gd, causal=causal, scale=scale)
    sdpa.check_device_error()
    sc = scale if scale != 0.0 else 1.0 / math.sqrt(d)
    rq, rk, rv = oracle.attn_bwd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                 dout.double().numpy(), sc, causal)
    return (dq, dk, dv), (rq, rk, rv)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,d,causal", [
    (1, 2, 2, 256, 256, 128, NONE),
    (1, 2, 2, 256, 256, 128, TL),
    (2, 4, 2, 200, 333, 64, NONE),     # GQA, ragged tails on both sides
    (2, 4, 2, 200, 333, 64, BR),
    (1, 2, 1, 300, 129, 128, BR),      # Sq > Sk: the first rows see no key
    (1, 2, 2, 129, 300, 128, TL),      # Sk > Sq: keys past Sq are seen by no row
    (1, 1, 1, 1, 1, 64, NONE),
    (1, 3, 1, 77, 77, 64, TL),
])
def test_bwd_matches_oracle(sdpa, B, Hq, Hkv, Sq, Sk, d, causal):
    (dq, dk, dv), (rq, rk, rv) = run_case(sdpa, B, Hq, Hkv, Sq, Sk, d, causal, seed=900 + Sq + Sk + causal)
    compare(dq, rq, "dq")
    compare(dk, rk, "dk")
    compare(dv, rv, "dv")


def test_bwd_masked_rows_and_unseen_keys_are_exact_zeros(sdpa):
    (dq, dk, dv), _ = run_case(sdpa, 1, 2, 1, 300, 129, 128, BR, seed=950)
    assert not dq[:, :, :171].any()  # rows i < Sq - Sk see no key (bottom-right)
    (dq, dk, dv), _ = run_case(sdpa, 1, 2, 2, 129, 300, 128, TL, seed=951)
    assert not dk[:, :, 129:].any() and not dv[:, :, 129:].any()


def test_bwd_explicit_scale(sdpa):
    (dq, dk, dv), (rq, rk, rv) = run_case(sdpa, 1, 2, 2, 192, 192, 128, NONE, seed=960, scale=0.05)
    compare(dq, rq, "dq")
    compare(dk, rk, "dk")
    compare(dv, rv, "dv")


def test_bwd_empty_sides(sdpa):
    dev = "cuda"
    q = torch.randn(1, 2, 0, 64, device=dev).bfloat16()
    k = torch.randn(1, 2, 5, 64, device=dev).bfloat16()
    v = torch.randn(1, 2, 5, 64, device=dev).bfloat16()
    o = torch.empty_like(q)
    lse = torch.empty(1, 2, 0, device=dev)
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(v, 7.0)
    _, dk, dv = sdpa.attn_bwd(q, k, v, o, lse, torch.empty_like(q), dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert not dk.any() and not dv.any()
    q = torch.randn(1, 2, 4, 64, device=dev).bfloat16()
    k = torch.randn(1, 2, 0, 64, device=dev).bfloat16()
    o, lse = sdpa.attn_fwd(q, k, k)
    dq = torch.full_like(q, 7.0)
    dq, _, _ = sdpa.attn_bwd(q, k, k, o, lse, torch.randn_like(q), dq=dq)
    torch.cuda.synchronize()
    assert not dq.any()
    sdpa.check_device_error()


@pytest.mark.parametrize("causal", [NONE, TL])
def test_bwd_full_sequence_length(sdpa, causal):
    """One head at the benchmark's sequence length (4096, d = 128), in the
    benchmark's launch configuration (per head the kernels do the same work
    at any batch); the oracle computes every gradient."""
    (dq, dk, dv), (rq, rk, rv) = run_case(sdpa, 1, 1, 1, 4096, 4096, 128, causal, seed=970 + causal)
    compare(dq, rq, "dq")
    compare(dk, rk, "dk")
    compare(dv, rv, "dv")
