"""GPU parity of the rotary-embedding / KV-cache append step
(``attn_rope_append``) against the fp64 oracle ``oracle.rope_append``.

Bar, per element: the kernel rotates in fp32 and rounds once to bf16, so
|gpu - ref| <= 2^-8 |ref| (bf16 round-to-nearest) + 2^-22 (|x_i| + |x_{i+d/2}|)
(fp32 products and sum of the rotation; the inputs are exact in fp32).  The v
rows are a copy (bit-exact), every cache row outside the appended range keeps
its bytes, and total_lens = past_lens + S_new exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from scaled_dot_product_fa2_b200 import _lib, inputs

pytestmark = pytest.mark.gpu

BHSD, BSHD = 0, 1


@pytest.fixture(scope="module")
def sdpa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scaled_dot_product_fa2_b200 import build
    build.build()
    import scaled_dot_product_fa2_b200 as m
    return m


def to_bhsd(cache, layout):
    return cache.transpose(1, 2) if layout == BSHD else cache


def rot_tolerance(packed, Hq, Hkv, d, heads):
    """Per-element bound for the rotated heads `heads` (a slice of head slots):
    2^-22 (|x_i| + |x_{i+d/2}|), shaped [B, S_new, n_heads, d]."""
    x = packed.double().numpy().reshape(packed.shape[0], packed.shape[1], Hq + 2 * Hkv, d)[:, :, heads]
    h = d // 2
    pair = np.abs(x[..., :h]) + np.abs(x[..., h:])
    return 2.0 ** -22 * np.concatenate([pair, pair], axis=-1)


def assert_close(gpu, ref, extra, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = 2.0 ** -8 * np.abs(ref) + extra
    worst = np.argmax(err - bound)
    assert (err <= bound).all(), f"{what}: |err| {err.flat[worst]:.3e} > bound {bound.flat[worst]:.3e}"


def run_case(sdpa, B, S_new, Hq, Hkv, d, cap, seed, layout=BHSD, past=None, max_pos=None):
    packed, kc, vc, past_lens = inputs.make_rope_inputs(B, S_new, Hq, Hkv, d, cap, seed, past, layout)
    cos, sin = inputs.rope_tables(max_pos or cap, d)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    q_shape = (B, S_new, Hq, d) if layout == BSHD else (B, Hq, S_new, d)
    q_d = torch.zeros(q_shape, dtype=torch.bfloat16, device="cuda")
    q_d, tot = sdpa.attn_rope_append(packed.cuda(), cos.cuda(), sin.cuda(), past_lens.cuda(), kc_d, vc_d, Hq, Hkv,
                                     layout=layout, q_out=q_d)
    torch.cuda.synchronize()
    return packed, kc, vc, past_lens, cos, sin, to_bhsd(q_d.cpu(), layout), to_bhsd(kc_d.cpu(), layout), \
        to_bhsd(vc_d.cpu(), layout), tot.cpu()


def check_against_oracle(sdpa, B, S_new, Hq, Hkv, d, cap, seed, layout=BHSD, past=None):
    packed, kc, vc, past_lens, cos, sin, q, kc_new, vc_new, tot = run_case(sdpa, B, S_new, Hq, Hkv, d, cap, seed,
                                                                           layout, past)
    sdpa.check_device_error()
    kc0, vc0 = to_bhsd(kc, layout), to_bhsd(vc, layout)
    q_ref, k_ref, v_ref, tot_ref = oracle.rope_append(packed.double().numpy(), cos.double().numpy(),
                                                      sin.double().numpy(), past_lens.numpy(),
                                                      kc0.double().numpy(), vc0.double().numpy(), Hq, Hkv)
    assert np.array_equal(tot.numpy(), tot_ref), "total_lens"
    assert_close(q.double().numpy(), q_ref, rot_tolerance(packed, Hq, Hkv, d, slice(0, Hq)).transpose(0, 2, 1, 3),
                 "q")
    k_extra = rot_tolerance(packed, Hq, Hkv, d, slice(Hq, Hq + Hkv)).transpose(0, 2, 1, 3)
    written = np.zeros((B, cap), dtype=bool)
    for b, p in enumerate(past_lens.tolist()):
        written[b, p:p + S_new] = True
        sl = slice(p, p + S_new)
        assert_close(kc_new[b, :, sl].double().numpy(), k_ref[b, :, sl], k_extra[b], f"k rows of batch {b}")
        # v is a copy: bit-exact
        assert torch.equal(vc_new[b, :, sl], torch.from_numpy(v_ref[b, :, sl]).bfloat16()), f"v rows of batch {b}"
    keep = torch.from_numpy(~written)[:, None, :, None].expand_as(kc_new)
    assert torch.equal(kc_new[keep], kc0[keep]), "k cache rows outside the appended range changed"
    assert torch.equal(vc_new[keep], vc0[keep]), "v cache rows outside the appended range changed"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,S_new,Hq,Hkv,cap", [
    (1, 1, 1, 1, 8),       # a single row per slot
    (3, 1, 8, 2, 40),      # decode step, GQA 4:1
    (2, 5, 4, 4, 16),      # several tokens, one sequence filled to capacity
    (4, 17, 6, 2, 64),     # odd token count: warps straddle tokens and slots
])
def test_rope_append_matches_oracle(sdpa, B, S_new, Hq, Hkv, cap, d):
    check_against_oracle(sdpa, B, S_new, Hq, Hkv, d, cap, seed=7100 + 7 * B + S_new + d)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_append_token_major_layout(sdpa, d):
    check_against_oracle(sdpa, 3, 6, 8, 4, d, 24, seed=7200 + d, layout=BSHD)


def test_rope_append_positions_far_into_the_table(sdpa):
    # large positions: the angles wrap many times; tables are read at past + t
    check_against_oracle(sdpa, 2, 3, 4, 2, 128, 3000, seed=7300, past=[2997, 1500])


def test_rope_append_out_of_range_positions_are_skipped_and_reported(sdpa):
    B, S_new, Hq, Hkv, d, cap = 3, 4, 4, 2, 64, 16
    # batch 0 runs 2 tokens past the end; batch 1 has a negative length; batch 2 is fine
    packed, kc, vc, past_lens, cos, sin, q, kc_new, vc_new, tot = run_case(sdpa, B, S_new, Hq, Hkv, d, cap, 7400,
                                                                           past=[cap - 2, -1, 3])
    with pytest.raises(_lib.AttnError) as e:
        sdpa.check_device_error()
    assert e.value.status == 13
    sdpa.check_device_error()  # the error word was cleared
    assert tot.tolist() == [cap + 2, 3, 7]
    # the in-range tokens of batch 0 and all of batch 2: the oracle on a cache with room for every token
    pad = lambda c: torch.cat([c, torch.zeros(B, Hkv, S_new, d, dtype=c.dtype)], dim=2)
    big_cos, big_sin = inputs.rope_tables(cap + S_new, d)
    assert torch.equal(big_cos[:cap], cos) and torch.equal(big_sin[:cap], sin)
    q_ref, k_ref, v_ref, _ = oracle.rope_append(packed.double().numpy(), big_cos.double().numpy(),
                                                big_sin.double().numpy(), np.array([cap - 2, 0, 3]),
                                                pad(kc).double().numpy(), pad(vc).double().numpy(), Hq, Hkv)
    qx = rot_tolerance(packed, Hq, Hkv, d, slice(0, Hq)).transpose(0, 2, 1, 3)
    kx = rot_tolerance(packed, Hq, Hkv, d, slice(Hq, Hq + Hkv)).transpose(0, 2, 1, 3)
    assert_close(q[0, :, :2].double().numpy(), q_ref[0, :, :2], qx[0, :, :2], "q of batch 0, in range")
    assert_close(q[2].double().numpy(), q_ref[2], qx[2], "q of batch 2")
    assert_close(kc_new[0, :, cap - 2:].double().numpy(), k_ref[0, :, cap - 2:cap], kx[0, :, :2], "k of batch 0")
    assert_close(kc_new[2, :, 3:7].double().numpy(), k_ref[2, :, 3:7], kx[2], "k of batch 2")
    # skipped rows write nothing: q stays as allocated (zeros), batch 1's cache keeps every byte
    assert not q[0, :, 2:].any() and not q[1].any()
    assert torch.equal(kc_new[1], kc[1]) and torch.equal(vc_new[1], vc[1])
    assert torch.equal(kc_new[0, :, :cap - 2], kc[0, :, :cap - 2])


def test_rope_append_lengths_advanced_in_place(sdpa):
    """total_lens may be past_lens itself (the decode loop's in-place update):
    every token must still be placed at its OLD length + t, across many blocks."""
    B, S_new, Hq, Hkv, d, cap = 8, 40, 8, 2, 128, 160
    packed, kc, vc, past_lens = inputs.make_rope_inputs(B, S_new, Hq, Hkv, d, cap, 7500)
    cos, sin = inputs.rope_tables(cap, d)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    lens_d = past_lens.cuda()
    q_d, tot = sdpa.attn_rope_append(packed.cuda(), cos.cuda(), sin.cuda(), lens_d, kc_d, vc_d, Hq, Hkv,
                                     total_lens=lens_d)
    sdpa.check_device_error()
    assert tot.data_ptr() == lens_d.data_ptr()
    q_ref, k_ref, v_ref, tot_ref = oracle.rope_append(packed.double().numpy(), cos.double().numpy(),
                                                      sin.double().numpy(), past_lens.numpy(),
                                                      kc.double().numpy(), vc.double().numpy(), Hq, Hkv)
    assert np.array_equal(lens_d.cpu().numpy(), tot_ref), "lengths advanced in place"
    assert_close(q_d.cpu().double().numpy(), q_ref,
                 rot_tolerance(packed, Hq, Hkv, d, slice(0, Hq)).transpose(0, 2, 1, 3), "q")
    k_extra = rot_tolerance(packed, Hq, Hkv, d, slice(Hq, Hq + Hkv)).transpose(0, 2, 1, 3)
    kc_new, vc_new = kc_d.cpu(), vc_d.cpu()
    for b, p in enumerate(past_lens.tolist()):
        sl = slice(p, p + S_new)
        assert_close(kc_new[b, :, sl].double().numpy(), k_ref[b, :, sl], k_extra[b], f"k rows of batch {b}")
        assert torch.equal(vc_new[b, :, sl], torch.from_numpy(v_ref[b, :, sl]).bfloat16()), f"v rows of batch {b}"


def test_rope_append_past_length_near_int_max_is_skipped(sdpa):
    """A corrupt past length near INT_MAX must not wrap into a negative
    position: its tokens are skipped and reported, its cache rows untouched,
    and its total length saturates at INT_MAX."""
    B, S_new, Hq, Hkv, d, cap = 2, 3, 4, 2, 128, 16
    big = 2 ** 31 - 2
    packed, kc, vc, past_lens, cos, sin, q, kc_new, vc_new, tot = run_case(sdpa, B, S_new, Hq, Hkv, d, cap, 7600,
                                                                           past=[big, 4])
    with pytest.raises(_lib.AttnError) as e:
        sdpa.check_device_error()
    assert e.value.status == 13
    sdpa.check_device_error()
    assert tot.tolist() == [2 ** 31 - 1, 7]
    assert not q[0].any(), "q rows of the skipped batch were written"
    assert torch.equal(kc_new[0], kc[0]) and torch.equal(vc_new[0], vc[0]), "cache of the skipped batch changed"
    q_ref, k_ref, _, _ = oracle.rope_append(packed[1:].double().numpy(), cos.double().numpy(), sin.double().numpy(),
                                            np.array([4]), kc[1:].double().numpy(), vc[1:].double().numpy(), Hq, Hkv)
    assert_close(q[1:].double().numpy(), q_ref,
                 rot_tolerance(packed[1:], Hq, Hkv, d, slice(0, Hq)).transpose(0, 2, 1, 3), "q of batch 1")


def test_rope_append_empty_inputs(sdpa):
    dev = "cuda"
    Hq, Hkv, d, cap = 4, 2, 64, 8
    cos, sin = (t.to(dev) for t in inputs.rope_tables(cap, d))
    kc = torch.randn(2, Hkv, cap, d, device=dev).bfloat16()
    vc = torch.randn(2, Hkv, cap, d, device=dev).bfloat16()
    k0, v0 = kc.clone(), vc.clone()
    past = torch.tensor([3, 5], dtype=torch.int32, device=dev)
    packed = torch.empty(2, 0, (Hq + 2 * Hkv) * d, dtype=torch.bfloat16, device=dev)
    q, tot = sdpa.attn_rope_append(packed, cos, sin, past, kc, vc, Hq, Hkv)
    torch.cuda.synchronize()
    assert q.shape == (2, Hq, 0, d) and tot.tolist() == [3, 5]
    assert torch.equal(kc, k0) and torch.equal(vc, v0)
    packed = torch.empty(0, 3, (Hq + 2 * Hkv) * d, dtype=torch.bfloat16, device=dev)
    q, tot = sdpa.attn_rope_append(packed, cos, sin, past[:0], kc[:0], vc[:0], Hq, Hkv)
    assert q.shape == (0, Hq, 3, d) and tot.shape == (0,)
    sdpa.check_device_error()


def test_rope_append_then_decode_reads_the_appended_rows(sdpa):
    """The total lengths feed the variable-length decode directly: attention of
    the rotated q over the updated cache equals the oracle's attention over the
    oracle's rotated q and cache."""
    B, S_new, Hq, Hkv, d, cap = 4, 1, 8, 2, 128, 512
    packed, kc, vc, past_lens, cos, sin, q, kc_new, vc_new, tot = run_case(sdpa, B, S_new, Hq, Hkv, d, cap, 7500)
    sdpa.check_device_error()
    o, lse = sdpa.attn_decode_splitkv_varlen(q.cuda(), kc_new.cuda(), vc_new.cuda(), tot.cuda(), causal=2)
    torch.cuda.synchronize()
    q_ref, k_ref, v_ref, tot_ref = oracle.rope_append(packed.double().numpy(), cos.double().numpy(),
                                                      sin.double().numpy(), past_lens.numpy(), kc.double().numpy(),
                                                      vc.double().numpy(), Hq, Hkv)
    for b in range(B):
        L = int(tot_ref[b])
        o_ref, lse_ref = oracle.attn_fwd(q_ref[b:b + 1], k_ref[b:b + 1, :, :L], v_ref[b:b + 1, :, :L],
                                         1.0 / np.sqrt(d), 2)
        # bf16 inputs on the GPU side vs fp64 on the oracle's: the attention bar
        assert np.abs(o[b].double().cpu().numpy() - o_ref[0]).max() <= 2e-2
        assert np.abs(lse[b].double().cpu().numpy() - lse_ref[0]).max() <= 1e-2


def test_rope_append_full_prompt_size_sampled(sdpa):
    """The prompt-size workload (8 x 4096 tokens, 16 + 2*16 heads, d = 128) in
    the launch the benchmark times; the oracle checks sampled tokens, each on
    its own (one token at its absolute position)."""
    w = inputs.ROPE_PROMPT
    packed, kc, vc, past_lens = inputs.make_rope_inputs(w.B, w.Sq, w.Hq, w.Hkv, w.d, w.Sk, w.seed,
                                                        past_lens=[0] * w.B)
    cos, sin = inputs.rope_tables(w.Sk, w.d)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    q_d, tot = sdpa.attn_rope_append(packed.cuda(), cos.cuda(), sin.cuda(), past_lens.cuda(), kc_d, vc_d, w.Hq, w.Hkv)
    sdpa.check_device_error()
    assert tot.cpu().tolist() == [w.Sq] * w.B
    rng = np.random.default_rng(7)
    picks = [(0, 0), (w.B - 1, w.Sq - 1), (3, 2048)] + [(int(rng.integers(w.B)), int(rng.integers(w.Sq)))
                                                       for _ in range(9)]
    for b, t in picks:
        zeros = np.zeros((1, w.Hkv, t + 1, w.d))
        q_ref, k_ref, v_ref, _ = oracle.rope_append(packed[b:b + 1, t:t + 1].double().numpy(),
                                                    cos.double().numpy(), sin.double().numpy(), [t], zeros, zeros,
                                                    w.Hq, w.Hkv)
        x = packed[b:b + 1, t:t + 1]
        qx = rot_tolerance(x, w.Hq, w.Hkv, w.d, slice(0, w.Hq))[0, 0]
        kx = rot_tolerance(x, w.Hq, w.Hkv, w.d, slice(w.Hq, w.Hq + w.Hkv))[0, 0]
        assert_close(q_d[b, :, t].double().cpu().numpy(), q_ref[0, :, 0], qx, f"q of token ({b}, {t})")
        assert_close(kc_d[b, :, t].double().cpu().numpy(), k_ref[0, :, t], kx, f"k of token ({b}, {t})")
        assert torch.equal(vc_d[b, :, t].cpu(), torch.from_numpy(v_ref[0, :, t]).bfloat16())
