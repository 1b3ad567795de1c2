"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's formula: each one checks a closed form,
an invariant, a hand-derived example or an independent brute force, chosen so
that a dropped term, a wrong sign or index, a transposed operand, a wrong
causal alignment or a wrong GQA mapping fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
NONE, TL, BR = 0, 1, 2


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _visible(causal, i, j, Sq, Sk):
    if causal == TL:
        return j <= i
    if causal == BR:
        return j <= i + Sk - Sq
    return True


def brute_force(q, k, v, scale, causal):
    """Independent scalar attention: nested loops, math.exp, math.fsum, no max
    subtraction (inputs are tiny, so exp cannot overflow)."""
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = [[[[0.0] * d for _ in range(Sq)] for _ in range(Hq)] for _ in range(B)]
    lse = [[[0.0] * Sq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for i in range(Sq):
                w = []
                for j in range(Sk):
                    if not _visible(causal, i, j, Sq, Sk):
                        continue
                    x = scale * math.fsum(float(q[b, h, i, c]) * float(k[b, hk, j, c])
                                          for c in range(d))
                    w.append((j, math.exp(x)))
                if not w:
                    lse[b][h][i] = -math.inf
                    continue
                z = math.fsum(e for _, e in w)
                lse[b][h][i] = math.log(z)
                for c in range(d):
                    o[b][h][i][c] = math.fsum(e * float(v[b, hk, j, c]) for j, e in w) / z
    return np.array(o), np.array(lse)


# ------------------------------------------------------------ hand-worked

def _ev(x):
    return float(eval(x, {"__builtins__": {}}, {"log": math.log, "inf": math.inf}))


def _arr(nested):
    if isinstance(nested, list):
        return [_arr(x) for x in nested]
    return _ev(nested)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_examples(oracle_mod, case):
    q, k, v = (np.array(_arr(case[n])) for n in ("q", "k", "v"))
    o_exp, lse_exp = np.array(_arr(case["o"])), np.array(_arr(case["lse"]))
    o, lse = oracle_mod.attn_fwd(q, k, v, _ev(case["scale"]), case["causal"])
    np.testing.assert_allclose(o, o_exp, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_exp))
    fin = np.isfinite(lse_exp)
    np.testing.assert_allclose(lse[fin], lse_exp[fin], rtol=0, atol=1e-12)


# ------------------------------------------------------------ brute force

TINY_SHAPES = list(itertools.product((1, 2, 3, 4), (1, 2, 3, 4), (1, 2, 3, 4), (1, 2),
                                     (NONE, TL, BR)))


def test_brute_force_every_tiny_shape(oracle_mod):
    """Every Sq, Sk in 1..4, d in 1..4, group size 1 or 2, each causal mode."""
    for n, (Sq, Sk, d, G, causal) in enumerate(TINY_SHAPES):
        Hkv = 2
        Hq = Hkv * G
        q = _rand((2, Hq, Sq, d), 10 * n)
        k = _rand((2, Hkv, Sk, d), 10 * n + 1)
        v = _rand((2, Hkv, Sk, d), 10 * n + 2)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle_mod.attn_fwd(q, k, v, scale, causal)
        ob, lseb = brute_force(q, k, v, scale, causal)
        assert not np.isnan(o).any()
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12,
                                   err_msg=f"Sq={Sq} Sk={Sk} d={d} G={G} causal={causal}")
        assert np.array_equal(np.isneginf(lse), np.isneginf(lseb))
        fin = np.isfinite(lseb)
        np.testing.assert_allclose(lse[fin], lseb[fin], rtol=0, atol=1e-12)


def test_probabilities_sum_to_one_and_match_exp(oracle_mod):
    """With v = identity (d = Sk) the output row IS the softmax row: it must sum
    to 1, vanish on masked keys and be proportional to exp(scale * q.k)."""
    Sk = 24
    Sq = 20
    for causal in (NONE, TL, BR):
        q = _rand((1, 1, Sq, Sk), 3)
        k = _rand((1, 1, Sk, Sk), 4)
        v = np.eye(Sk)[None, None]
        scale = 0.3
        p, lse = oracle_mod.attn_fwd(q, k, v, scale, causal)
        p = p[0, 0]
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
        x = scale * (q[0, 0] @ k[0, 0].T)
        for i in range(Sq):
            vis = np.array([_visible(causal, i, j, Sq, Sk) for j in range(Sk)])
            assert np.all(p[i, ~vis] == 0.0)
            np.testing.assert_allclose(p[i, vis], np.exp(x[i, vis] - lse[0, 0, i]),
                                       rtol=1e-12, atol=0)


# ----------------------------------------------------- closed forms / invariants

def test_causal_row0_is_v0(oracle_mod):
    q = _rand((2, 3, 50, 16), 5)
    k = _rand((2, 3, 50, 16), 6)
    v = _rand((2, 3, 50, 16), 7)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.25, TL)
    assert np.array_equal(o[:, :, 0, :], v[:, :, 0, :])
    np.testing.assert_allclose(lse[:, :, 0], 0.25 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [NONE, TL, BR])
def test_zero_query_gives_prefix_mean(oracle_mod, causal):
    """q = 0 makes every score 0: each row averages the V rows it may see and
    lse = log(count)."""
    Sq, Sk, d = 37, 53, 8
    if causal == TL:
        Sq = Sk  # keep every row non-empty
    q = np.zeros((1, 2, Sq, d))
    k = _rand((1, 2, Sk, d), 8)
    v = _rand((1, 2, Sk, d), 9)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.7, causal)
    for i in range(Sq):
        cnt = sum(_visible(causal, i, j, Sq, Sk) for j in range(Sk))
        np.testing.assert_allclose(o[:, :, i], v[:, :, :cnt].mean(axis=2), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], math.log(cnt), rtol=0, atol=1e-12)


def test_single_key_returns_v0(oracle_mod):
    q = _rand((2, 2, 9, 32), 10)
    k = _rand((2, 2, 1, 32), 11)
    v = _rand((2, 2, 1, 32), 12)
    o, _ = oracle_mod.attn_fwd(q, k, v, 0.1, NONE)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-15)


def test_identical_keys_give_mean_of_visible_v(oracle_mod):
    Sq = Sk = 31
    q = _rand((1, 1, Sq, 8), 13) * 5.0
    k = np.broadcast_to(_rand((1, 1, 1, 8), 14), (1, 1, Sk, 8)).copy()
    v = _rand((1, 1, Sk, 8), 15)
    o, _ = oracle_mod.attn_fwd(q, k, v, 1.0, TL)
    for i in range(Sq):
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, :i + 1].mean(axis=0), rtol=0, atol=1e-12)


def test_noncausal_permutation_invariance(oracle_mod):
    q = _rand((1, 2, 17, 16), 16)
    k = _rand((1, 2, 40, 16), 17)
    v = _rand((1, 2, 40, 16), 18)
    perm = np.random.default_rng(0).permutation(40)
    o1, l1 = oracle_mod.attn_fwd(q, k, v, 0.25, NONE)
    o2, l2 = oracle_mod.attn_fwd(q, k[:, :, perm], v[:, :, perm], 0.25, NONE)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_score_shift_invariance(oracle_mod):
    """Append a dimension with q=1 and k=c: every score moves by scale*c, so O is
    unchanged and lse moves by scale*c."""
    q = _rand((1, 1, 12, 8), 19)
    k = _rand((1, 1, 12, 8), 20)
    v = _rand((1, 1, 12, 8), 21)
    c, scale = 3.5, 0.5
    q2 = np.concatenate([q, np.ones((1, 1, 12, 1))], axis=-1)
    k2 = np.concatenate([k, np.full((1, 1, 12, 1), c)], axis=-1)
    v2 = np.concatenate([v, np.zeros((1, 1, 12, 1))], axis=-1)
    for causal in (NONE, TL):
        o1, l1 = oracle_mod.attn_fwd(q, k, v, scale, causal)
        o2, l2 = oracle_mod.attn_fwd(q2, k2, v2, scale, causal)
        np.testing.assert_allclose(o1, o2[..., :8], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1 + scale * c, l2, rtol=0, atol=1e-12)


def test_scale_multiplies_scores(oracle_mod):
    q = _rand((1, 2, 10, 8), 22)
    k = _rand((1, 2, 10, 8), 23)
    v = _rand((1, 2, 10, 8), 24)
    o1, l1 = oracle_mod.attn_fwd(q, k, v, 2.0, TL)
    o2, l2 = oracle_mod.attn_fwd(2.0 * q, k, v, 1.0, TL)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [NONE, TL, BR])
def test_gqa_equals_explicit_expansion(oracle_mod, causal):
    Hq, Hkv = 8, 2
    q = _rand((2, Hq, 11, 8), 25)
    k = _rand((2, Hkv, 14, 8), 26)
    v = _rand((2, Hkv, 14, 8), 27)
    o1, l1 = oracle_mod.attn_fwd(q, k, v, 0.3, causal)
    G = Hq // Hkv
    o2, l2 = oracle_mod.attn_fwd(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), 0.3, causal)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # and a wrong mapping (hq % Hkv) would differ
    o3, _ = oracle_mod.attn_fwd(q, np.tile(k, (1, G, 1, 1)), np.tile(v, (1, G, 1, 1)), 0.3, causal)
    assert np.abs(o1 - o3).max() > 1e-3


def test_rows_api_matches_full(oracle_mod):
    q = _rand((2, 4, 19, 16), 28)
    k = _rand((2, 2, 23, 16), 29)
    v = _rand((2, 2, 23, 16), 30)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.25, BR)
    rows = np.array([0, 5, 18, 19, 75, 2 * 4 * 19 - 1])
    orow, lrow = oracle_mod.attn_rows(q, k, v, 0.25, BR, rows)
    np.testing.assert_array_equal(orow, o.reshape(-1, 16)[rows])
    np.testing.assert_array_equal(lrow, lse.reshape(-1)[rows])


# ------------------------------------------------------- FA2 recurrence pin

@pytest.mark.parametrize("bk", [1, 3, 128])
@pytest.mark.parametrize("causal", [NONE, TL, BR])
def test_online_recurrence_equals_definition(oracle_mod, causal, bk):
    """The FlashAttention-2 loop (running max/sum, one final division) reaches
    the plain five-step result for any key-block size."""
    q = _rand((1, 2, 45, 16), 31) * 2.0
    k = _rand((1, 2, 70, 16), 32) * 2.0
    v = _rand((1, 2, 70, 16), 33)
    o1, l1 = oracle_mod.attn_fwd(q, k, v, 0.4, causal)
    o2, l2 = oracle_mod.online_attn(q, k, v, 0.4, causal, block_q=7, block_k=bk)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


# ------------------------------------------------------- split-KV combine pin

def _bounds(Sk, ns):
    return [round(s * Sk / ns) for s in range(ns + 1)]


@pytest.mark.parametrize("ns", [1, 2, 3, 7, 61])
@pytest.mark.parametrize("causal", [NONE, BR])
def test_split_combine_equals_unsplit(oracle_mod, ns, causal):
    """Locally normalised partials rescaled by their (max, sum) metadata give
    exactly full softmax.V (the decode reduce step)."""
    Sq, Sk = 4, 61
    q = _rand((2, 8, Sq, 16), 34) * 2.0
    k = _rand((2, 2, Sk, 16), 35) * 2.0
    v = _rand((2, 2, Sk, 16), 36)
    o1, l1 = oracle_mod.attn_fwd(q, k, v, 0.35, causal)
    po, pm, pl = oracle_mod.split_partials(q, k, v, 0.35, causal, _bounds(Sk, ns))
    o2, l2 = oracle_mod.split_combine(po, pm, pl)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_split_with_masked_and_empty_splits(oracle_mod):
    """Bottom-right mask with Sq > Sk: some splits see nothing (weight 0) and
    some rows see nothing at all (o = 0, lse = -inf)."""
    Sq, Sk = 9, 6
    q = _rand((1, 2, Sq, 8), 37)
    k = _rand((1, 1, Sk, 8), 38)
    v = _rand((1, 1, Sk, 8), 39)
    o1, l1 = oracle_mod.attn_fwd(q, k, v, 0.5, BR)
    po, pm, pl = oracle_mod.split_partials(q, k, v, 0.5, BR, [0, 2, 2, 5, 6])
    assert (pl == 0).any()
    o2, l2 = oracle_mod.split_combine(po, pm, pl)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(l1), np.isneginf(l2))
    assert np.isneginf(l1).any() and not np.isnan(o1).any()
    fin = np.isfinite(l1)
    np.testing.assert_allclose(l1[fin], l2[fin], rtol=0, atol=1e-12)


def test_partials_are_locally_normalised(oracle_mod):
    """Each split's partial is softmax over that split's keys alone (the fused
    decode kernel's local normalisation)."""
    q = _rand((1, 1, 1, 8), 40)
    k = _rand((1, 1, 10, 8), 41)
    v = _rand((1, 1, 10, 8), 42)
    po, pm, pl = oracle_mod.split_partials(q, k, v, 0.5, NONE, [0, 4, 10])
    o_a, l_a = oracle_mod.attn_fwd(q, k[:, :, :4], v[:, :, :4], 0.5, NONE)
    np.testing.assert_allclose(po[0, 0, 0, 0], o_a[0, 0, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(pm[0, 0, 0, 0] + math.log(pl[0, 0, 0, 0]), l_a[0, 0, 0], atol=1e-12)


# --------------------------------------------------------------- additive bias
# ("[onnxruntime] WebGPU FlashAttention: kernel fusion ...", section 1: the
# fused decode applies an attention bias with the mask; its two leading dims
# broadcast over batch and heads.)

def brute_force_bias(q, k, v, bias, scale, causal):
    """Independent scalar attention with an additive bias on the scaled scores."""
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Sq, d))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            bb, bh = (0 if bias.shape[0] == 1 else b), (0 if bias.shape[1] == 1 else h)
            for i in range(Sq):
                w = []
                for j in range(Sk):
                    if not _visible(causal, i, j, Sq, Sk):
                        continue
                    x = scale * math.fsum(float(q[b, h, i, c]) * float(k[b, hk, j, c]) for c in range(d))
                    w.append((j, math.exp(x + float(bias[bb, bh, i, j]))))
                w = [(j, e) for j, e in w if e > 0.0]
                if not w:
                    lse[b, h, i] = -math.inf
                    continue
                z = math.fsum(e for _, e in w)
                lse[b, h, i] = math.log(z)
                for c in range(d):
                    o[b, h, i, c] = math.fsum(e * float(v[b, hk, j, c]) for j, e in w) / z
    return o, lse


@pytest.mark.parametrize("dims", [(1, 1), (2, 1), (1, 4), (2, 4)])
@pytest.mark.parametrize("causal", [NONE, TL, BR])
def test_bias_brute_force_every_broadcast(oracle_mod, dims, causal):
    B, Hq, Hkv, Sq, Sk, d = 2, 4, 2, 3, 5, 3
    q, k, v = _rand((B, Hq, Sq, d), 1), _rand((B, Hkv, Sk, d), 2), _rand((B, Hkv, Sk, d), 3)
    bias = _rand((dims[0], dims[1], Sq, Sk), 4)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.7, causal, bias=bias)
    o_bf, lse_bf = brute_force_bias(q, k, v, bias, 0.7, causal)
    assert np.allclose(o, o_bf, atol=1e-12, rtol=0)
    assert np.allclose(lse, lse_bf, atol=1e-12, rtol=0)


def test_bias_of_log_weights_with_zero_query_is_weighted_mean(oracle_mod):
    """q = 0 makes every score 0, so bias_j = log w_j gives softmax weights
    w_j / sum w: o = sum_j w_j v_j / sum_j w_j and lse = log sum_j w_j (a closed
    form; a bias that were subtracted, scaled or applied after the softmax
    fails it)."""
    B, H, Sq, Sk, d = 1, 2, 3, 6, 4
    q = np.zeros((B, H, Sq, d))
    k, v = _rand((B, H, Sk, d), 5), _rand((B, H, Sk, d), 6)
    w = np.random.default_rng(7).uniform(0.1, 3.0, size=(B, H, Sq, Sk))
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.9, NONE, bias=np.log(w))
    expect = np.einsum("bhij,bhjc->bhic", w, v) / w.sum(-1, keepdims=True)
    assert np.allclose(o, expect, atol=1e-12)
    assert np.allclose(lse, np.log(w.sum(-1)), atol=1e-12)


def test_constant_bias_per_row_shifts_lse_only(oracle_mod):
    """Adding c_i to every score of row i leaves the softmax unchanged and adds
    c_i to the row's LSE."""
    B, Hq, Hkv, Sq, Sk, d = 1, 2, 1, 4, 9, 5
    q, k, v = _rand((B, Hq, Sq, d), 8), _rand((B, Hkv, Sk, d), 9), _rand((B, Hkv, Sk, d), 10)
    c = _rand((1, Hq, Sq, 1), 11) * 5.0
    for causal in (NONE, BR):
        o0, l0 = oracle_mod.attn_fwd(q, k, v, 0.4, causal)
        o1, l1 = oracle_mod.attn_fwd(q, k, v, 0.4, causal, bias=np.broadcast_to(c, (1, Hq, Sq, Sk)))
        assert np.allclose(o1, o0, atol=1e-12)
        assert np.allclose(l1, l0 + c[..., 0], atol=1e-12)


def test_minus_infinity_bias_masks_keys(oracle_mod):
    """A -inf bias on a key is the same as removing that key; a row whose keys
    are all -inf gives o = 0 and lse = -inf."""
    B, H, Sq, Sk, d = 1, 1, 3, 6, 4
    q, k, v = _rand((B, H, Sq, d), 12), _rand((B, H, Sk, d), 13), _rand((B, H, Sk, d), 14)
    keep = np.array([0, 2, 5])
    bias = np.full((1, 1, Sq, Sk), -np.inf)
    bias[..., keep] = 0.0
    bias[0, 0, 2, :] = -np.inf
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.6, NONE, bias=bias)
    o_ref, lse_ref = oracle_mod.attn_fwd(q[:, :, :2], k[:, :, keep], v[:, :, keep], 0.6, NONE)
    assert np.allclose(o[:, :, :2], o_ref, atol=1e-12)
    assert np.allclose(lse[:, :, :2], lse_ref, atol=1e-12)
    assert np.all(o[0, 0, 2] == 0.0) and lse[0, 0, 2] == -np.inf


def test_bias_rows_api_matches_full(oracle_mod):
    B, Hq, Hkv, Sq, Sk, d = 2, 2, 1, 5, 7, 3
    q, k, v = _rand((B, Hq, Sq, d), 15), _rand((B, Hkv, Sk, d), 16), _rand((B, Hkv, Sk, d), 17)
    bias = _rand((B, 1, Sq, Sk), 18)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, TL, bias=bias)
    rows = np.array([0, 3, 7, 12, 19])
    o_r, l_r = oracle_mod.attn_rows(q, k, v, 0.5, TL, rows, bias=bias)
    assert np.allclose(o_r, o.reshape(-1, d)[rows], atol=1e-13)
    assert np.allclose(l_r, lse.reshape(-1)[rows], atol=1e-13)


# ------------------------------------------------------ rotary + KV append
# (the fused split / rotary / copy-KV step named by the decode page, section 2;
# reading: non-interleaved rotary embedding)

def _rope_tables(max_pos, d, base=10000.0):
    inv = base ** (-np.arange(0, d // 2) * 2.0 / d)
    ang = np.arange(max_pos)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def test_rope_relative_position_property(oracle_mod):
    """RoPE's defining property: the rotated q.k depends only on the distance
    between the two positions (shifting both positions leaves it unchanged),
    and equals the plain q.k at distance 0."""
    d, cap = 8, 64
    cos, sin = _rope_tables(cap, d)
    rng = np.random.default_rng(20)
    qv, kv = rng.standard_normal(d), rng.standard_normal(d)

    def rotated_dot(pq, pk):
        packed_q = np.zeros((1, 1, 3 * d))
        packed_q[0, 0, :d] = qv
        packed_q[0, 0, d:2 * d] = kv
        qa, ka, _, _ = oracle_mod.rope_append(packed_q, cos, sin, [pq], np.zeros((1, 1, cap, d)),
                                              np.zeros((1, 1, cap, d)), 1, 1)
        packed_k = packed_q.copy()
        _, kb, _, _ = oracle_mod.rope_append(packed_k, cos, sin, [pk], np.zeros((1, 1, cap, d)),
                                             np.zeros((1, 1, cap, d)), 1, 1)
        return float(qa[0, 0, 0] @ kb[0, 0, pk])

    assert abs(rotated_dot(5, 5) - float(qv @ kv)) < 1e-12
    for dist in (0, 1, 3, 7):
        ref = rotated_dot(10 + dist, 10)
        for shift in (0, 4, 20):
            assert abs(rotated_dot(10 + dist + shift, 10 + shift) - ref) < 1e-10
    # and it does change with distance (the rotation is not the identity)
    assert abs(rotated_dot(13, 10) - rotated_dot(10, 10)) > 1e-3


def test_rope_append_positions_norms_and_untouched_rows(oracle_mod):
    """Position 0 is the identity; every (i, i + d/2) pair keeps its norm;
    v rows are copied unrotated to rows past .. past + S_new - 1, the other
    cache rows are unchanged, and the total lengths are past + S_new."""
    B, S_new, Hq, Hkv, d, cap = 2, 3, 4, 2, 8, 16
    cos, sin = _rope_tables(cap, d)
    rng = np.random.default_rng(21)
    packed = rng.standard_normal((B, S_new, (Hq + 2 * Hkv) * d))
    kc0, vc0 = rng.standard_normal((B, Hkv, cap, d)), rng.standard_normal((B, Hkv, cap, d))
    past = [0, 9]
    q, kc, vc, tot = oracle_mod.rope_append(packed, cos, sin, past, kc0, vc0, Hq, Hkv)
    assert list(tot) == [3, 12]
    half = d // 2
    # batch 0, token 0 sits at position 0: no rotation
    assert np.allclose(q[0, :, 0], packed[0, 0, :Hq * d].reshape(Hq, d), atol=0)
    for b in range(B):
        for s in range(S_new):
            pos = past[b] + s
            for h in range(Hq):
                x = packed[b, s, h * d:(h + 1) * d]
                y = q[b, h, s]
                assert np.allclose(np.hypot(y[:half], y[half:]), np.hypot(x[:half], x[half:]), atol=1e-12)
            for h in range(Hkv):
                assert np.array_equal(vc[b, h, pos], packed[b, s, (Hq + Hkv + h) * d:(Hq + Hkv + h + 1) * d])
        rows = [r for r in range(cap) if not past[b] <= r < past[b] + S_new]
        assert np.array_equal(kc[b][:, rows], kc0[b][:, rows]) and np.array_equal(vc[b][:, rows], vc0[b][:, rows])


def test_rope_quarter_turn_closed_form(oracle_mod):
    """With cos = 0, sin = 1 (a quarter turn) the pair (a, b) becomes (-b, a)."""
    d, cap = 4, 2
    cos, sin = np.zeros((cap, d // 2)), np.ones((cap, d // 2))
    packed = np.arange(1, 3 * d + 1, dtype=float).reshape(1, 1, 3 * d)
    q, kc, _, _ = oracle_mod.rope_append(packed, cos, sin, [1], np.zeros((1, 1, cap, d)),
                                         np.zeros((1, 1, cap, d)), 1, 1)
    assert np.array_equal(q[0, 0, 0], np.array([-3.0, -4.0, 1.0, 2.0]))
    assert np.array_equal(kc[0, 0, 1], np.array([-7.0, -8.0, 5.0, 6.0]))


# ------------------------------------------------------------ backward pass
# (the pages give no backward algorithm; the oracle is the chain rule through
# the five naive steps, pinned here by finite differences of the forward
# oracle and by properties of the softmax Jacobian)

def _bwd_inputs(B, Hq, Hkv, Sq, Sk, d, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Hq, Sq, d)), rng.standard_normal((B, Hkv, Sk, d)),
            rng.standard_normal((B, Hkv, Sk, d)), rng.standard_normal((B, Hq, Sq, d)))


@pytest.mark.parametrize("causal", [0, 1, 2])
@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,d", [(1, 1, 1, 3, 4, 3), (2, 2, 1, 4, 3, 2), (1, 2, 2, 5, 5, 4)])
def test_bwd_matches_finite_differences(oracle_mod, B, Hq, Hkv, Sq, Sk, d, causal):
    """Every entry of dq, dk, dv equals the central difference of
    L = sum(o * dout) through the forward oracle (h = 1e-5: truncation and
    rounding errors both below 1e-9)."""
    q, k, v, g = _bwd_inputs(B, Hq, Hkv, Sq, Sk, d, 100 + causal)
    scale = 0.6
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, scale, causal)
    loss = lambda qq, kk, vv: float((oracle_mod.attn_fwd(qq, kk, vv, scale, causal)[0] * g).sum())
    h = 1e-5
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        base = [q, k, v]
        for idx in np.ndindex(*base[which].shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd = (loss(*plus) - loss(*minus)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-8, (which, idx, fd, grad[idx])


def test_bwd_single_key_closed_form(oracle_mod):
    """With one key every output row is v_0: dv_0 sums dout over all rows of
    every query head of the group, and q and k get no gradient."""
    q, k, v, g = _bwd_inputs(2, 4, 2, 5, 1, 3, 110)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, 0.5, 0)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    for b in range(2):
        for hk in range(2):
            expect = g[b, 2 * hk:2 * hk + 2].sum(axis=(0, 1))
            assert np.allclose(dv[b, hk, 0], expect, atol=1e-12)


@pytest.mark.parametrize("causal", [0, 1, 2])
def test_bwd_key_gradients_sum_to_zero_and_key_shift_leaves_dq(oracle_mod, causal):
    """Each row of the softmax Jacobian sums to zero, so sum_j dk_j = 0; and
    adding one vector to every key shifts a row's scores by a constant, so o
    and dq do not change."""
    q, k, v, g = _bwd_inputs(2, 2, 1, 6, 6, 4, 120 + causal)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, 0.8, causal)
    assert np.abs(dk.sum(axis=2)).max() < 1e-12
    shift = np.random.default_rng(5).standard_normal(4)
    dq2, _, _ = oracle_mod.attn_bwd(q, k + shift, v, g, 0.8, causal)
    assert np.abs(dq2 - dq).max() < 1e-10


@pytest.mark.parametrize("causal", [0, 1, 2])
def test_bwd_gqa_equals_explicit_expansion(oracle_mod, causal):
    """dk, dv of a shared KV head = the sum over its query heads of the
    gradients with K/V repeated per query head."""
    q, k, v, g = _bwd_inputs(1, 4, 2, 5, 6, 3, 130 + causal)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, 0.7, causal)
    ke, ve = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dqe, dke, dve = oracle_mod.attn_bwd(q, ke, ve, g, 0.7, causal)
    assert np.allclose(dq, dqe, atol=1e-12)
    assert np.allclose(dk, dke.reshape(1, 2, 2, 6, 3).sum(axis=2), atol=1e-12)
    assert np.allclose(dv, dve.reshape(1, 2, 2, 6, 3).sum(axis=2), atol=1e-12)


def test_bwd_masked_rows_and_unseen_keys_get_no_gradient(oracle_mod):
    """Bottom-right with Sq > Sk: the first Sq - Sk rows see no key, so their
    dq is 0.  Top-left with Sk > Sq: keys j >= Sq are seen by no row, so their
    dk and dv are 0."""
    q, k, v, g = _bwd_inputs(1, 1, 1, 6, 3, 4, 140)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, 0.5, 2)
    assert np.array_equal(dq[0, 0, :3], np.zeros((3, 4)))
    assert np.abs(dq[0, 0, 3:]).max() > 0
    q, k, v, g = _bwd_inputs(1, 1, 1, 3, 6, 4, 141)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, 0.5, 1)
    assert np.array_equal(dk[0, 0, 3:], np.zeros((3, 4))) and np.array_equal(dv[0, 0, 3:], np.zeros((3, 4)))


def test_bwd_two_key_closed_form(oracle_mod):
    """One query, two keys, d = 1, derived by hand: with x_j = s q k_j,
    P = softmax(x), o = P1 v1 + P2 v2 and dout = g,
      dv_j = P_j g,  dx_1 = -dx_2 = P1 P2 g (v1 - v2),
      dq = s dx_1 (k1 - k2),  dk_1 = -dk_2 = s dx_1 q."""
    q, k1, k2, v1, v2, g, s = 0.7, -1.3, 0.4, 2.0, -0.5, 1.7, 0.9
    e1, e2 = np.exp(s * q * k1), np.exp(s * q * k2)
    P1, P2 = e1 / (e1 + e2), e2 / (e1 + e2)
    dx1 = P1 * P2 * g * (v1 - v2)
    dq, dk, dv = oracle_mod.attn_bwd(np.array([[[[q]]]]), np.array([[[[k1], [k2]]]]), np.array([[[[v1], [v2]]]]),
                                     np.array([[[[g]]]]), s, 0)
    assert abs(dq[0, 0, 0, 0] - s * dx1 * (k1 - k2)) < 1e-14
    assert abs(dk[0, 0, 0, 0] - s * dx1 * q) < 1e-14 and abs(dk[0, 0, 1, 0] + s * dx1 * q) < 1e-14
    assert abs(dv[0, 0, 0, 0] - P1 * g) < 1e-14 and abs(dv[0, 0, 1, 0] - P2 * g) < 1e-14
