"""The bounded-wait contract on the GPU: a kernel whose wait runs out returns
(no trap, no hang), the host reads ATTN_ERR_DEVICE_TIMEOUT from
``attn_check_device_error``, and the context stays usable.

The wait is made to run out the accepted way -- a flag that nothing sets:
``attn_selftest_decode_wait_timeout`` runs the split-KV decode kernel with its
K/V copies withheld, so its consumer warps wait on "stage filled" barriers no
copy will ever complete.  That kernel holds no tensor memory and, in this
mode, has no copy in flight when it gives up.
"""
import math

import pytest
import torch

from scaled_dot_product_fa2_b200 import _lib
from tests import parity

pytestmark = pytest.mark.gpu

BR = 2


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scaled_dot_product_fa2_b200 import build
    build.build()
    import scaled_dot_product_fa2_b200 as m
    return m


def test_wait_that_runs_out_is_reported_and_the_context_survives(sdpa):
    B, Hq, Hkv, Sq, Sk, d = 1, 4, 1, 1, 256, 128
    q, k, v = parity.seeded(B, Hq, Hkv, Sq, Sk, d, seed=900)
    qd, kd, vd = parity.to_dev(q, k, v)
    o = torch.empty_like(qd)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
    ws = sdpa.decode_workspace(qd, kd)
    lib = _lib.get()
    stream = torch.cuda.current_stream().cuda_stream
    sdpa.check_device_error()  # start from a clear error word
    st = lib.attn_selftest_decode_wait_timeout(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                                               lse.data_ptr(), B, Hq, Hkv, Sq, Sk, d, ws.data_ptr(),
                                               ws.numel(), stream)
    assert st == 0  # the launch itself succeeds; the failure is reported by the device
    with pytest.raises(_lib.AttnError) as err:
        sdpa.check_device_error()
    assert err.value.status == 9  # ATTN_ERR_DEVICE_TIMEOUT
    sdpa.check_device_error()  # the word was cleared by the read
    # the context is intact: the same decode, loads included, matches the oracle
    o2, lse2 = sdpa.attn_decode_splitkv(qd, kd, vd, causal=BR, workspace=ws)
    sdpa.check_device_error()
    o_ref, lse_ref = parity.oracle_full(q, k, v, 1 / math.sqrt(d), BR)
    parity.compare(o2.float().cpu().numpy(), lse2.cpu().numpy(), o_ref, lse_ref, "after timeout")
