"""The allocation-free decode entry point, ``attn_decode_splitkv_static``.

It serves callers that cannot give the library device memory (a plug-in whose
host framework owns all allocations, a service with a budget fixed at
start-up): the split partials live in the library's own fixed 16 MiB device
array instead of a caller workspace.  Its results must match the workspace
entry point ``attn_decode_splitkv`` on the same inputs, call after call, even
though every call reuses (and leaves behind) the same scratch contents.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from tests import parity

NONE, TL, BR = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    from scaled_dot_product_fa2_b200 import _lib, build
    build.build()
    return _lib.get()


def _call_static(lib, q, k, v, o, lse, causal, num_splits=0):
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    return lib.attn_decode_splitkv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                          B, Hq, Hkv, Sq, Sk, d, 0.0, causal, num_splits,
                                          torch.cuda.current_stream().cuda_stream)


def _call_workspace(lib, q, k, v, o, lse, causal, num_splits=0):
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    n = lib.attn_decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, num_splits)
    ws = torch.empty(n, dtype=torch.uint8, device=q.device)
    return lib.attn_decode_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   B, Hq, Hkv, Sq, Sk, d, 0.0, causal, num_splits, ws.data_ptr(), n,
                                   torch.cuda.current_stream().cuda_stream), ws


def _dirty_scratch(lib):
    """A larger problem with another split count through the static entry, so
    the next static call runs over stale partials of a different layout."""
    q, k, v = parity.to_dev(*parity.seeded(2, 16, 4, 4, 3000, 128, 303))
    o = torch.empty_like(q)
    lse = torch.empty((2, 16, 4), dtype=torch.float32, device="cuda")
    assert _call_static(lib, q, k, v, o, lse, BR, num_splits=11) == 0


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_two_calls_in_a_row(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    shapes = [
        # B, Hq, Hkv, Sq, Sk, d, causal, seed: two different problems back to back,
        # so the second call runs over the first call's leftover scratch
        (2, 8, 2, 4, 4096, 128, BR, 101),
        (1, 4, 1, 1, 1000, 128, BR, 202),
    ]
    for B, Hq, Hkv, Sq, Sk, d, causal, seed in shapes:
        q, k, v = parity.to_dev(*parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed))
        o_ref = torch.empty_like(q)
        lse_ref = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
        st, ws = _call_workspace(lib, q, k, v, o_ref, lse_ref, causal)
        assert st == 0
        for _ in range(2):
            _dirty_scratch(lib)
            o = torch.empty_like(q)
            lse = torch.empty_like(lse_ref)
            assert _call_static(lib, q, k, v, o, lse, causal) == 0
            assert lib.attn_check_device_error(torch.cuda.current_stream().cuda_stream) == 0
            # the same kernels with the same split count on the same inputs:
            # identical bits, whatever the scratch held before
            assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        err = (o.float() - o_ref.float()).abs()
        assert err.max().item() <= parity.O_MAX_ERR and err.mean().item() <= parity.O_MEAN_ERR
        assert (lse - lse_ref).abs().max().item() <= parity.LSE_ERR
        del ws


@pytest.mark.gpu
def test_static_scratch_rejects_problems_beyond_its_size(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q = torch.zeros(8, 32, 16, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(8, 8, 8192, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(8, 32, 16, dtype=torch.float32, device="cuda")
    need = lib.attn_decode_workspace_size(8, 32, 8, 16, 8192, 128, 128)
    assert need > 16 << 20
    assert _call_static(lib, q, k, k, o, lse, BR, num_splits=128) == 12  # ATTN_ERR_SCRATCH_LIMIT
    assert lib.attn_status_string(12)
