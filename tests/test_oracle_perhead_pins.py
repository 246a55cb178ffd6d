"""Pins of the oracle's per-head-indexer-key variant (no GPU needed).

Each of the 4 indexer heads has its own projection W_h (w_idx [512][4][64]) and its own FP4 key
per entry; head h's dot uses key h.  The pins tie it to the base reading (one key shared by the
heads, which is the variant with W_h = W for every h), to exact rational arithmetic on tiny
inputs, to a head-permutation symmetry, to brute-force top-k and to append = prefill.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth


def _perhead_w(w, heads=4):
    """[512,64] -> [512,4,64] with the same W for every head."""
    return np.repeat(np.asarray(w, np.float32)[:, None, :], heads, axis=1).copy()


def test_identical_heads_reduce_to_the_shared_key(orc):
    inp = synth.prefill_inputs(4 * 40 + 3, seed=51)
    bits = synth.bits16(inp["raw"])
    gate, bias, w = inp["gate"].numpy(), inp["bias4"].numpy(), inp["w_idx"].numpy()
    kv0, ik0, is0 = orc.compress(bits, gate, bias, 4, w)
    kv1, ik1, is1 = orc.compress_perhead(bits, gate, bias, 4, _perhead_w(w))
    assert np.array_equal(kv0, kv1)
    for h in range(4):
        assert np.array_equal(ik1[:, h], ik0) and np.array_equal(is1[:, h], is0)
    rng = np.random.default_rng(52)
    q = rng.standard_normal((4, 64)).astype(np.float32)
    hw = np.abs(rng.standard_normal(4)).astype(np.float32)
    a32, a64 = orc.indexer_scores(ik0, is0, q, hw)
    b32, b64 = orc.indexer_scores_perhead(ik1, is1, q, hw)
    assert np.array_equal(a32, b32) and np.array_equal(a64, b64)


def test_perhead_keys_are_each_heads_projection(orc):
    inp = synth.prefill_inputs(4 * 6, seed=53)
    bits = synth.bits16(inp["raw"])
    gate, bias = inp["gate"].numpy(), inp["bias4"].numpy()
    rng = np.random.default_rng(54)
    w = (rng.standard_normal((512, 4, 64)) / np.sqrt(512)).astype(np.float32)
    _, ik, isc = orc.compress_perhead(bits, gate, bias, 4, w)
    for s in range(6):
        c = orc.pool_block(bits[4 * s:4 * s + 4], gate[4 * s:4 * s + 4], bias)
        u = orc.indexer_key_raw_perhead(c, w)
        for h in range(4):
            assert np.allclose(u[h], orc.indexer_key_raw(c, w[:, h, :].copy()), rtol=0, atol=1e-12)
            codes, scales = orc.fp4_quantize64(u[h])
            assert np.array_equal(ik[s, h], codes) and np.array_equal(isc[s, h], scales)


def test_perhead_scores_exact(orc):
    g = synth.gen(55)
    rng = np.random.default_rng(56)
    n = 48
    keys = np.zeros((n, 4, 32), np.uint8)
    scales = np.zeros((n, 4, 2), np.float32)
    for h in range(4):
        ik, isc = synth.random_ikeys(1, n, g, heavy_frac=0.1)
        keys[:, h], scales[:, h] = ik[0].numpy(), isc[0].numpy()
    q = rng.standard_normal((4, 64)).astype(np.float32)
    hw = np.abs(rng.standard_normal(4)).astype(np.float32)
    hw[1] = -hw[1]
    s32, s64 = orc.indexer_scores_perhead(keys, scales, q, hw)
    qd = []
    for h in range(4):
        c, s = orc.fp4_quantize64(q[h].astype(np.float64))
        qd.append([Fraction(v) for v in orc.fp4_dequantize64(c, s)])
    for i in range(n):
        e, mag = Fraction(0), Fraction(0)
        for h in range(4):
            kd = [Fraction(v) for v in orc.fp4_dequantize64(keys[i, h], scales[i, h])]
            dot = sum(a * b for a, b in zip(qd[h], kd))
            term = Fraction(float(hw[h])) * max(dot, Fraction(0))
            e += term
            mag += abs(term)
        assert abs(Fraction(s64[i]) - e) <= mag * Fraction(1, 10 ** 14)
        assert abs(Fraction(float(s32[i])) - e) <= 4 * mag / 2 ** 24


def test_head_permutation_symmetry(orc):
    """Permuting the heads of the keys, the queries and the head weights together leaves every
    fp64 score unchanged."""
    g = synth.gen(57)
    rng = np.random.default_rng(58)
    n = 100
    keys = np.zeros((n, 4, 32), np.uint8)
    scales = np.zeros((n, 4, 2), np.float32)
    for h in range(4):
        ik, isc = synth.random_ikeys(1, n, g)
        keys[:, h], scales[:, h] = ik[0].numpy(), isc[0].numpy()
    q = rng.standard_normal((4, 64)).astype(np.float32)
    hw = np.abs(rng.standard_normal(4)).astype(np.float32)
    perm = [2, 0, 3, 1]
    _, a = orc.indexer_scores_perhead(keys, scales, q, hw)
    _, b = orc.indexer_scores_perhead(keys[:, perm].copy(), scales[:, perm].copy(), q[perm].copy(), hw[perm].copy())
    assert np.allclose(a, b, rtol=1e-14, atol=0)


def test_perhead_topk_batch_is_bruteforce(orc):
    g = synth.gen(59)
    rng = np.random.default_rng(60)
    B, cap, k = 3, 500, 37
    keys = np.zeros((B, cap, 4, 32), np.uint8)
    scales = np.zeros((B, cap, 4, 2), np.float32)
    for h in range(4):
        ik, isc = synth.random_ikeys(B, cap, g)
        keys[:, :, h], scales[:, :, h] = ik.numpy(), isc.numpy()
    q = rng.standard_normal((B, 4, 64)).astype(np.float32)
    hw = np.abs(rng.standard_normal((B, 4))).astype(np.float32)
    seq = np.array([4 * cap, 4 * 300 + 3, 4 * 20], np.int32)
    got = orc.indexer_topk_batch_perhead(keys, scales, seq, 4, q, hw, k)
    for b in range(B):
        n = min(seq[b] // 4, cap)
        s32, _ = orc.indexer_scores_perhead(keys[b, :n], scales[b, :n], q[b], hw[b])
        order = sorted(range(n), key=lambda i: (-float(s32[i]), i))[:k]
        want = sorted(order) + [-1] * (k - len(order))
        assert list(got[b]) == want


def test_append_perhead_equals_prefill_perhead(orc):
    T, W = 4 * 70 + 3, 16
    inp = synth.prefill_inputs(T, seed=61)
    bits = synth.bits16(inp["raw"])
    gate, bias = inp["gate"].numpy(), inp["bias4"].numpy()
    rng = np.random.default_rng(62)
    w = (rng.standard_normal((512, 4, 64)) / np.sqrt(512)).astype(np.float32)
    kv, ik, isc = orc.compress_perhead(bits, gate, bias, 4, w)
    E = T // 4
    st = orc.LayerState(1, E + 1, 4, W, True, key_heads=4)
    for t in range(T):
        orc.append_batch(st, bias, w, bits[t:t + 1], gate[t:t + 1])
    assert np.array_equal(st.comp_kv[0, :E], kv)
    assert np.array_equal(st.ikeys[0, :E], ik) and np.array_equal(st.iscales[0, :E], isc)
