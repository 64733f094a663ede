"""Pins of the CPU fp64 oracle to facts that do not come from the oracle.

Every oracle function is checked here against at least one of: a hand-derived
worked example (tests/golden/), a closed form, brute-force loops on tiny
inputs, torch's own CPU attention, or an invariant of the method (any
chunking of K/V equals one-shot attention; the Ulysses all-to-all followed by
its inverse is the identity).  ``test_planted_mistakes_are_caught`` plants
plausible mistakes in copies of the oracle and checks that these pins fail.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from context_attention_dits_cp_b200 import workloads as wl

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _qkv(B, H, Sq, Skv, D, seed):
    return _rand((B, Sq, H, D), seed), _rand((B, Skv, H, D), seed + 1), _rand((B, Skv, H, D), seed + 2)


# ---------------------------------------------------------------- worked examples
def test_golden_two_key_attention():
    g = json.load(open(os.path.join(GOLD, "two_key_example.json")))
    out, lse = oracle.attention(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]), g["scale"])
    np.testing.assert_allclose(out[0, 0, 0], g["out"], rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - g["lse"]) < 1e-15


def test_golden_two_key_chunk_partials_and_merge():
    g = json.load(open(os.path.join(GOLD, "two_key_example.json")))
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    oa, la = oracle.attention_partial(q, k[:, :1], v[:, :1], g["scale"])
    ob, lb = oracle.attention_partial(q, k[:, 1:], v[:, 1:], g["scale"])
    np.testing.assert_allclose(oa[0, 0, 0], g["out_A"], atol=0)
    np.testing.assert_allclose(ob[0, 0, 0], g["out_B"], atol=0)
    assert la[0, 0, 0] == g["lse_A"] and lb[0, 0, 0] == g["lse_B"]
    for (o1, l1, o2, l2) in ((oa, la, ob, lb), (ob, lb, oa, la)):
        o, l = oracle.lse_merge(o1, l1, o2, l2)
        np.testing.assert_allclose(o[0, 0, 0], g["out"], atol=1e-15)
        assert abs(l[0, 0, 0] - g["lse"]) < 1e-15


def test_golden_ring_chunks():
    g = json.load(open(os.path.join(GOLD, "ring_chunks.json")))
    for c in g["cases"]:
        offs = oracle.ring_chunk_offsets(c["S"], c["R"])
        assert list(np.diff(offs)) == c["lengths"]
        # the input generator's own split must agree with the oracle's
        assert wl.ring_chunk_lengths(c["S"], c["R"]) == c["lengths"]


def test_golden_ulysses_index_map():
    g = json.load(open(os.path.join(GOLD, "ulysses_index_map.json")))
    x = np.array(g["x"]).reshape(g["x_shape"])
    y = np.array(g["y"]).reshape(g["y_shape"])
    assert np.array_equal(oracle.ulysses_permute(x, g["degree"], 0), y)
    assert np.array_equal(oracle.ulysses_permute(y, g["degree"], 1), x)


# ---------------------------------------------------------------- brute force / library
@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (2, 3, 5, 7, 4), (1, 2, 9, 3, 8)])
@pytest.mark.parametrize("scale", [None, 0.37])
def test_bruteforce_tiny(shape, scale):
    B, H, Sq, Skv, D = shape
    q, k, v = _qkv(B, H, Sq, Skv, D, 7)
    o1, l1 = oracle.attention(q, k, v, scale)
    o2, l2 = oracle.attention_bruteforce(q, k, v, scale)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


@pytest.mark.parametrize("shape", [(2, 3, 64, 80, 16), (1, 2, 700, 300, 32)])
def test_torch_sdpa_fp64(shape):
    """torch's CPU scaled_dot_product_attention (fp64) is an independent
    implementation of the same definition; it also crosses the 512-row
    block boundary of the oracle."""
    B, H, Sq, Skv, D = shape
    q, k, v = _qkv(B, H, Sq, Skv, D, 11)
    o, _ = oracle.attention(q, k, v)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)   # BSHD -> BHSD
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms
def test_constant_v_returns_v():
    q, k, _ = _qkv(2, 3, 17, 23, 8, 3)
    c = _rand((8,), 4)
    v = np.broadcast_to(c, (2, 23, 3, 8)).copy()
    o, _ = oracle.attention(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-13)


def test_zero_q_gives_mean_and_log_n():
    _, k, v = _qkv(1, 2, 5, 37, 8, 5)
    q = np.zeros((1, 5, 2, 8))
    o, l = oracle.attention(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape), atol=1e-14)
    np.testing.assert_allclose(l, math.log(37), atol=1e-14)


def test_single_dominant_key():
    """k_{j*} = alpha * q: its score dwarfs the others, so out -> v_{j*} and
    lse -> s_{j*} (the remainder is below fp64 resolution)."""
    rng = np.random.default_rng(9)
    D, S = 16, 40
    q = rng.standard_normal((1, 1, 1, D))
    k = rng.standard_normal((1, S, 1, D)) * 0.1
    v = rng.standard_normal((1, S, 1, D))
    js = 13
    k[0, js, 0] = 400.0 * q[0, 0, 0]
    o, l = oracle.attention(q, k, v, scale=1.0)
    s_star = 400.0 * float(q[0, 0, 0] @ q[0, 0, 0])
    np.testing.assert_allclose(o[0, 0, 0], v[0, js, 0], atol=1e-12)
    assert abs(l[0, 0, 0] - s_star) < 1e-9


def test_scale_enters_lse_linearly_for_equal_scores():
    """All keys equal: every score is scale*q.k, so lse = scale*q.k + ln S_kv."""
    rng = np.random.default_rng(10)
    q = rng.standard_normal((1, 3, 1, 8))
    k = np.broadcast_to(rng.standard_normal(8), (1, 6, 1, 8)).copy()
    v = rng.standard_normal((1, 6, 1, 8))
    for sc in (0.25, 1.0, 3.0):
        _, l = oracle.attention(q, k, v, sc)
        np.testing.assert_allclose(l[0, 0], sc * (q[0, :, 0] @ k[0, 0, 0]) + math.log(6), atol=1e-13)


def test_empty_keys_is_merge_identity():
    q = _rand((1, 4, 2, 8), 1)
    e = np.zeros((1, 0, 2, 8))
    o, l = oracle.attention(q, e, e)
    assert np.all(o == 0) and np.all(np.isneginf(l))


# ---------------------------------------------------------------- merge / ring invariants
def test_merge_identities():
    q, k, v = _qkv(1, 2, 9, 11, 8, 21)
    o, l = oracle.attention(q, k, v)
    zo, zl = np.zeros_like(o), np.full_like(l, -np.inf)
    for (a, b) in (((o, l), (zo, zl)), ((zo, zl), (o, l))):
        mo, ml = oracle.lse_merge(*a, *b)
        assert np.array_equal(mo, o) and np.array_equal(ml, l)
    mo, ml = oracle.lse_merge(o, l, o, l)
    np.testing.assert_allclose(mo, o, atol=1e-15)
    np.testing.assert_allclose(ml, l + math.log(2), atol=1e-14)
    mo, ml = oracle.lse_merge(zo, zl, zo, zl)
    assert np.all(mo == 0) and np.all(np.isneginf(ml))


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
def test_any_even_chunking_equals_oneshot(R):
    q, k, v = _qkv(2, 3, 19, 41, 8, 30 + R)
    o, l = oracle.attention(q, k, v)
    offs = oracle.ring_chunk_offsets(41, R)
    n = len(offs) - 1
    for rot in range(n):
        order = [(rot + i) % n for i in range(n)]
        ro, rl = oracle.ring_attention(q, k, v, offs, order=order)
        np.testing.assert_allclose(ro, o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(rl, l, rtol=0, atol=1e-13)


def test_random_uneven_chunking_with_empty_chunks():
    rng = np.random.default_rng(77)
    q, k, v = _qkv(1, 2, 13, 50, 8, 40)
    o, l = oracle.attention(q, k, v)
    for _ in range(10):
        cuts = sorted(rng.integers(0, 51, size=rng.integers(1, 7)).tolist())
        offs = [0] + cuts + [50]
        order = rng.permutation(len(offs) - 1).tolist()
        ro, rl = oracle.ring_attention(q, k, v, offs, order=order)
        np.testing.assert_allclose(ro, o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(rl, l, rtol=0, atol=1e-13)


def test_ring_degree_one_is_plain_attention_exactly():
    q, k, v = _qkv(1, 2, 13, 29, 8, 50)
    o, l = oracle.attention(q, k, v)
    ro, rl = oracle.ring_attention(q, k, v, [0, 29])
    assert np.array_equal(ro, o) and np.array_equal(rl, l)


def test_padding_beyond_a_chunk_never_contributes():
    """Ring Anything trims padded K/V; a partial over a chunk must not read
    past it: poisoned rows after the chunk leave the partial unchanged."""
    q, k, v = _qkv(1, 1, 4, 12, 8, 60)
    o, l = oracle.attention_partial(q, k[:, :7], v[:, :7])
    kp, vp = k.copy(), v.copy()
    kp[:, 7:] = np.nan
    vp[:, 7:] = 1e30
    o2, l2 = oracle.attention_partial(q, kp[:, :7], vp[:, :7])
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


# ---------------------------------------------------------------- Ulysses / unified
@pytest.mark.parametrize("U,B,S,H,D", [(2, 1, 4, 2, 3), (3, 2, 6, 6, 2), (4, 1, 8, 8, 1)])
def test_ulysses_bruteforce_and_inverse(U, B, S, H, D):
    x = np.arange(U * B * (S // U) * H * D, dtype=np.int64).reshape(U, B, S // U, H, D)
    y = oracle.ulysses_permute(x, U, 0)
    assert np.array_equal(y, oracle.ulysses_permute_bruteforce(x, U, 0))
    assert np.array_equal(oracle.ulysses_permute(y, U, 1), x)
    assert np.array_equal(oracle.ulysses_permute_bruteforce(y, U, 1), x)
    # every element moves exactly once
    assert sorted(y.ravel().tolist()) == list(range(x.size))


def test_ulysses_bits_preserved_bf16():
    U = 4
    x = torch.randn(U, 2, 8, 8, 16).to(torch.bfloat16).view(torch.int16).numpy()
    y = oracle.ulysses_permute(x, U, 0)
    assert np.array_equal(oracle.ulysses_permute(y, U, 1), x)


@pytest.mark.parametrize("R,U", [(1, 4), (2, 2), (4, 1), (2, 3)])
def test_usp_equals_oneshot(R, U):
    B, S, H, D = 2, 48, 12, 8
    q, k, v = _qkv(B, H, S, S, D, 90 + R * 10 + U)
    o, l = oracle.attention(q, k, v)
    sh = lambda x: x.reshape(B, R * U, S // (R * U), H, D).transpose(1, 0, 2, 3, 4)
    uo, ul = oracle.usp_attention(sh(q), sh(k), sh(v), R, U)
    np.testing.assert_allclose(uo, sh(o), rtol=0, atol=1e-13)
    np.testing.assert_allclose(ul, l, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- planted mistakes
def _pins_pass(att, merge):
    """A compact battery of the pins above, run against a candidate pair."""
    g = json.load(open(os.path.join(GOLD, "two_key_example.json")))
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    try:
        o, l = att(q, k, v, g["scale"])
        if not (np.allclose(o[0, 0, 0], g["out"], atol=1e-12) and abs(l[0, 0, 0] - g["lse"]) < 1e-12):
            return False
        q, k, v = _qkv(1, 2, 5, 7, 3, 123)        # S_q != S_kv != D catches transposes
        o, l = att(q, k, v, 0.37)
        ob, lb = oracle.attention_bruteforce(q, k, v, 0.37)
        if not (np.allclose(o, ob, atol=1e-12) and np.allclose(l, lb, atol=1e-12)):
            return False
        oa, la = att(q, k[:, :3], v[:, :3], 0.37)
        oc, lc = att(q, k[:, 3:], v[:, 3:], 0.37)
        mo, ml = merge(oa, la, oc, lc)
        return bool(np.allclose(mo, ob, atol=1e-12) and np.allclose(ml, lb, atol=1e-12))
    except Exception:
        return False


def test_planted_mistakes_are_caught():
    assert _pins_pass(oracle.attention, oracle.lse_merge)

    def no_scale(q, k, v, scale=None):
        return oracle.attention(q, k, v, 1.0)

    def log2_lse(q, k, v, scale=None):
        o, l = oracle.attention(q, k, v, scale)
        return o, l / math.log(2)

    def unnormalised(q, k, v, scale=None):
        o, l = oracle.attention(q, k, v, scale)
        return o * np.exp(l - l.max()).transpose(0, 2, 1)[..., None], l

    def k_for_v(q, k, v, scale=None):
        return oracle.attention(q, k, k, scale)

    def merge_wrong_sign(oa, la, ob, lb):
        m = np.maximum(la, lb)
        new = m - np.log1p(np.exp(-np.abs(la - lb)))
        wa = np.exp(la - new).transpose(0, 2, 1)[..., None]
        wb = np.exp(lb - new).transpose(0, 2, 1)[..., None]
        return wa * oa + wb * ob, new

    def merge_drop_weight(oa, la, ob, lb):
        o, l = oracle.lse_merge(oa, la, ob, lb)
        return 0.5 * (oa + ob), l

    for bad in (no_scale, log2_lse, unnormalised, k_for_v):
        assert not _pins_pass(bad, oracle.lse_merge), bad.__name__
    for bad in (merge_wrong_sign, merge_drop_weight):
        assert not _pins_pass(oracle.attention, bad), bad.__name__


def test_planted_permute_mistake_is_caught():
    g = json.load(open(os.path.join(GOLD, "ulysses_index_map.json")))
    x = np.array(g["x"]).reshape(g["x_shape"])
    y = np.array(g["y"]).reshape(g["y_shape"])

    def head_major_wrong(x, U, d):       # takes heads strided instead of contiguous
        Uu, B, Sl, H, D = x.shape
        return np.stack([np.concatenate([x[p][:, :, q::U] for p in range(U)], axis=1)
                         for q in range(U)])

    def shard_order_swapped(x, U, d):
        return oracle.ulysses_permute(x[::-1], U, d)

    assert np.array_equal(oracle.ulysses_permute(x, 2, 0), y)
    assert not np.array_equal(shard_order_swapped(x, 2, 0), y)
    x3 = np.arange(2 * 1 * 2 * 4 * 1).reshape(2, 1, 2, 4, 1)
    assert not np.array_equal(head_major_wrong(x3, 2, 0), oracle.ulysses_permute_bruteforce(x3, 2, 0))


# ---------------------------------------------------------------- Ulysses Anything
def _flat_shards(full, offs):
    """Rank buffers of a [B, S, H, D] array split at `offs`, concatenated."""
    return np.concatenate([full[:, offs[p]:offs[p + 1]].reshape(-1) for p in range(len(offs) - 1)])


def test_uneven_offsets_rule():
    assert oracle.uneven_offsets(4481, 4) == [0, 1121, 2242, 3363, 4481]
    assert oracle.uneven_offsets(24, 5) == [0, 5, 10, 15, 20, 24]
    assert oracle.uneven_offsets(3, 4) == [0, 1, 2, 3, 3]


def test_ulysses_anything_reduces_to_even_map():
    """With even splits the flat rank buffers are exactly the rank-major
    tensors of the even all-to-all, so both maps must agree bit for bit."""
    U, B, S, H, D = 4, 2, 16, 8, 3
    x = np.arange(B * S * H * D).reshape(B, S, H, D)
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    flat = _flat_shards(x, so)
    even = x.reshape(B, U, S // U, H, D).transpose(1, 0, 2, 3, 4)
    y = oracle.ulysses_anything_permute(flat, B, H, D, so, ho, 0)
    assert np.array_equal(y, oracle.ulysses_permute(even, U, 0).reshape(-1))


@pytest.mark.parametrize("U,B,S,H,D", [(4, 1, 13, 6, 2), (5, 2, 11, 24, 1), (3, 1, 7, 4, 3)])
def test_ulysses_anything_bruteforce_and_inverse(U, B, S, H, D):
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    full = np.arange(B * S * H * D).reshape(B, S, H, D)
    x = _flat_shards(full, so)
    y = oracle.ulysses_anything_permute(x, B, H, D, so, ho, 0)
    # element by element: rank q holds every token of its heads, in order
    pos = 0
    for q in range(U):
        for b in range(B):
            for t in range(S):
                for h in range(ho[q], ho[q + 1]):
                    for d in range(D):
                        assert y[pos] == full[b, t, h, d]
                        pos += 1
    assert np.array_equal(oracle.ulysses_anything_permute(y, B, H, D, so, ho, 1), x)


@pytest.mark.parametrize("U,S,H", [(4, 37, 8), (5, 23, 24), (3, 19, 7)])
def test_ulysses_anything_attention_equals_oneshot(U, S, H):
    B, D = 2, 8
    q, k, v = _qkv(B, H, S, S, D, 200 + U)
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    out, lse = oracle.ulysses_anything_attention(_flat_shards(q, so), _flat_shards(k, so),
                                                 _flat_shards(v, so), B, H, D, so, ho)
    o, l = oracle.attention(q, k, v)
    np.testing.assert_allclose(out, _flat_shards(o, so), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, l, rtol=0, atol=1e-13)
