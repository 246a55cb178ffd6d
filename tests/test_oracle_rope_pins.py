"""Pins of the oracle's RoPE-at-compressed-positions variant (no GPU needed).

The variant rotates the 64 RoPE dims of each entry (dims 448..511, kept in bf16 by the pages'
storage paragraph) at the entry's own position: RoFormer's rotation of consecutive pairs,
pair i = dims (448 + 2i, 449 + 2i) turned by pos * base^(-i/32); a compressed entry s of
ratio m at its block's last token pos0 + (s+1) m - 1, a window entry at its own token.  The
pins below tie it to closed forms (the first pair's frequency is 1, pair 16's is base^(-1/2)),
to the properties that define a rotary encoding (identity at 0, composition, the score of two
rotated vectors depending only on their position difference, norms kept) and to the base
reading (m = 1 pooling is the identity; W_I blind to the RoPE dims gives the base keys;
token-by-token append reproduces the prefill).
"""
import math

import numpy as np
import pytest
import torch

import synth

BASE = 10000.0


def _rand512(rng):
    return rng.standard_normal(512)


def test_rope_zero_position_is_identity(orc):
    rng = np.random.default_rng(1)
    x = _rand512(rng)
    assert np.array_equal(orc.rope_rotate(x, 0, BASE), x)


def test_rope_pair_frequencies_closed_form(orc):
    """Pair 0 turns by 1 rad per position; pair 16 by base^(-1/2) = 0.01 rad (so 100 positions
    turn it by 1 rad); pair 31 by base^(-31/32).  A unit vector stays inside its own pair of
    consecutive dims (interleaved pairs, not halves)."""
    for dim, pos, angle in ((448, 1, 1.0), (480, 100, 1.0), (510, 1000, 1000.0 * BASE ** (-31 / 32)),
                            (449, 3, 3.0)):
        x = np.zeros(512)
        x[dim] = 1.0
        y = orc.rope_rotate(x, pos, BASE)
        lo = dim - (dim - 448) % 2
        if dim == lo:   # e_{2i} -> (cos a, sin a)
            want = (math.cos(angle), math.sin(angle))
        else:           # e_{2i+1} -> (-sin a, cos a)
            want = (-math.sin(angle), math.cos(angle))
        assert abs(y[lo] - want[0]) < 1e-12 and abs(y[lo + 1] - want[1]) < 1e-12, (dim, y[lo:lo + 2])
        others = np.delete(y, [lo, lo + 1])
        assert not others.any(), dim


def test_rope_composition_and_norms(orc):
    rng = np.random.default_rng(2)
    x = _rand512(rng)
    for a, b in ((3, 5), (1000, 24), (262143, 1)):
        ab = orc.rope_rotate(orc.rope_rotate(x, a, BASE), b, BASE)
        direct = orc.rope_rotate(x, a + b, BASE)
        assert np.allclose(ab, direct, rtol=0, atol=1e-9)
        y = orc.rope_rotate(x, a, BASE)
        pairs_x = np.hypot(x[448::2], x[449::2])
        pairs_y = np.hypot(y[448::2], y[449::2])
        assert np.allclose(pairs_x, pairs_y, rtol=1e-13, atol=0)
        assert np.array_equal(y[:448], x[:448])          # the E4M3 dims are never rotated


def test_rope_score_depends_only_on_position_difference(orc):
    """<R(a) u, R(b) v> over the RoPE dims equals <R(a - b) u, v>: what makes it relative."""
    rng = np.random.default_rng(3)
    u, v = _rand512(rng), _rand512(rng)
    for a, b in ((10, 3), (1 << 20, (1 << 20) - 5), (7, 7)):
        lhs = float(orc.rope_rotate(u, a, BASE)[448:] @ orc.rope_rotate(v, b, BASE)[448:])
        rhs = float(orc.rope_rotate(u, a - b, BASE)[448:] @ v[448:])
        assert abs(lhs - rhs) < 1e-9 * max(1.0, abs(rhs)) * (1 + math.log2(1 + a)), (a, b, lhs, rhs)


def test_compress_rope_ratio_one_rotates_each_token_at_its_position(orc):
    """m = 1: pooling is the identity, so entry s is raw token s rotated at pos0 + s."""
    rng = np.random.default_rng(4)
    T, pos0 = 37, 123456
    raw = rng.standard_normal((T, 512)).astype(np.float32)
    bits = (raw.view(np.uint32) >> 16).astype(np.uint16)
    x = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    gate = rng.standard_normal(T).astype(np.float32)
    kv, _, _ = orc.compress_rope(bits, gate, np.zeros(1, np.float32), 1, pos0, BASE)
    for s in range(T):
        assert np.array_equal(kv[s], orc.entry_encode(orc.rope_rotate(x[s], pos0 + s, BASE))), s


def test_compress_rope_entry_position_is_block_last_token(orc):
    """Entry s of ratio m is the base entry's pooled vector rotated at pos0 + (s+1) m - 1: the
    E4M3 bytes equal the base compressor's, and undoing that rotation on the stored RoPE dims
    gives back the base entry's bf16 values within one bf16 step."""
    inp = synth.prefill_inputs(4 * 9 + 3, seed=31)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"].numpy()
    pos0 = 5000
    kv, _, _ = orc.compress(bits, gate, bias, 4)
    kvr, _, _ = orc.compress_rope(bits, gate, bias, 4, pos0, BASE)
    assert np.array_equal(kv[:, :448], kvr[:, :448])
    for s in range(kv.shape[0]):
        back = orc.rope_rotate(orc.entry_decode(kvr[s]), -(pos0 + 4 * s + 3), BASE)
        base = orc.entry_decode(kv[s])
        err = np.abs(back[448:] - base[448:])
        assert (err <= 2.0 ** -7 * np.abs(base[448:]).max() + 1e-30).all(), s
        wrong = orc.rope_rotate(orc.entry_decode(kvr[s]), -(pos0 + 4 * s), BASE)
        assert np.abs(wrong[448:] - base[448:]).max() > 2.0 ** -6 * np.abs(base[448:]).max(), s


def test_compress_rope_keys_follow_the_rotated_vector(orc):
    """W_I blind to the RoPE dims: the keys are the base keys.  W_I reading only the RoPE dims:
    the keys are those of the rotated vector (they differ from the base keys)."""
    inp = synth.prefill_inputs(64, seed=32)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"].numpy()
    w = inp["w_idx"].numpy().copy()
    w_nope = w.copy()
    w_nope[448:] = 0.0
    _, ik0, is0 = orc.compress(bits, gate, bias, 4, w_nope)
    _, ik1, is1 = orc.compress_rope(bits, gate, bias, 4, 777, BASE, w_nope)
    assert np.array_equal(ik0, ik1) and np.array_equal(is0, is1)
    w_rope = w.copy()
    w_rope[:448] = 0.0
    _, ik2, _ = orc.compress_rope(bits, gate, bias, 4, 777, BASE, w_rope)
    _, ik3, _ = orc.compress(bits, gate, bias, 4, w_rope)
    assert not np.array_equal(ik2, ik3)
    # the key of entry 0 is FP4 of (pooled vector, rotated at 777 + 3) . W_I
    c = orc.rope_rotate(orc.pool_block(bits[:4], gate[:4], bias), 780, BASE)
    codes, scales = orc.fp4_quantize64(orc.indexer_key_raw(c, w_rope))
    assert np.array_equal(codes, ik2[0])


@pytest.mark.parametrize("m,W,idx", [(4, 16, True), (128, 32, False)])
def test_append_rope_equals_prefill_rope(orc, m, W, idx):
    """Token-by-token append with RoPE reproduces the RoPE prefill (pos0 = 0), and its window
    entries are the tokens rotated at their own positions."""
    T = 2 * 128 + 37
    inp = synth.prefill_inputs(T, seed=33)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"].numpy() if m == 4 else inp["bias128"].numpy()
    w_idx = inp["w_idx"].numpy() if idx else None
    kv, ik, isc = orc.compress_rope(bits, gate, bias, m, 0, BASE, w_idx)
    E = T // m
    st = orc.LayerState(1, E + 1, m, W, idx)
    for t in range(T):
        orc.append_batch(st, bias, w_idx, bits[t:t + 1], gate[t:t + 1], rope_base=BASE)
    assert np.array_equal(st.comp_kv[0, :E], kv)
    if idx:
        assert np.array_equal(st.ikeys[0, :E], ik) and np.array_equal(st.iscales[0, :E], isc)
    raw64 = inp["raw"].to(torch.float64).numpy()
    for t in range(T - W, T):
        assert np.array_equal(st.win_kv[0, t % W], orc.entry_encode(orc.rope_rotate(raw64[t], t, BASE)))
