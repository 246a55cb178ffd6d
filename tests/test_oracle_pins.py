"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to a library routine, a closed form, brute force on a tiny
input, an invariant of the mathematics, or a figure printed on the pages (tests/golden/), so
that a dropped term, a wrong sign or index, or a transposed operand in the oracle fails here.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------
# Codecs: E4M3, bf16 and E2M1, against torch's own dtype casts and the format definitions.
# ------------------------------------------------------------------------------------------
def test_e4m3_decode_all_codes_match_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = orc.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c]), c


def test_e4m3_encode_roundtrip_and_midpoints(orc):
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    for c in finite:
        assert orc.e4m3_encode(orc.e4m3_decode(c)) == c
    # midpoints between neighbouring positive codes go to the even code (mantissa lsb 0)
    for c in range(0, 0x7E):
        lo, hi = orc.e4m3_decode(c), orc.e4m3_decode(c + 1)
        mid = 0.5 * (lo + hi)
        want = c if (c & 1) == 0 else c + 1
        assert orc.e4m3_encode(mid) == want, (c, mid)
        assert orc.e4m3_encode(-mid) == (want | 0x80)
        # just off the midpoint goes to the nearer code
        assert orc.e4m3_encode(mid - (hi - lo) * 1e-6) == c
        assert orc.e4m3_encode(mid + (hi - lo) * 1e-6) == c + 1
    # saturation (no infinities in E4M3): anything at or beyond 448 becomes +-448
    for v in (448.0, 460.0, 479.0, 1e4, 1e30):
        assert orc.e4m3_encode(v) == 0x7E and orc.e4m3_encode(-v) == 0xFE


def test_e4m3_encode_matches_torch_cast(orc):
    g = torch.Generator().manual_seed(1)
    x = torch.randn(20000, generator=g) * torch.exp2(torch.randint(-12, 8, (20000,), generator=g).float())
    x = x.clamp(-470, 470)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(v)) for v in x.tolist()], np.uint8)
    assert np.array_equal(got, ref)


def test_bf16_codec_matches_torch(orc):
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    sample = np.concatenate([np.arange(0, 65536, 97), np.array([0x0001, 0x007F, 0x0080, 0x7F7F, 0x8001])])
    for c in sample:
        r = ref[c]
        got = orc.bf16_decode(int(c))
        if math.isnan(r):
            assert math.isnan(got)
        else:
            assert got == r
    g = torch.Generator().manual_seed(2)
    x = torch.randn(20000, generator=g) * torch.exp2(torch.randint(-130, 120, (20000,), generator=g).float())
    refb = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_encode(float(v)) for v in x.tolist()], np.uint16)
    assert np.array_equal(got, refb)


def test_e2m1_grid_and_ties(orc):
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = orc.e2m1_decode(c)
        assert abs(v) == grid[c & 7] and (v < 0) == (c >= 8 and grid[c & 7] > 0)
        assert orc.e2m1_encode(v) == (c if c != 8 else 8)
    # round-to-nearest-even on the grid: ties go to the even mantissa code
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        assert orc.e2m1_decode(orc.e2m1_encode(x)) == want
        assert orc.e2m1_decode(orc.e2m1_encode(-x)) == -want
    for x, want in {0.26: 0.5, 0.74: 0.5, 2.4: 2.0, 2.6: 3.0, 4.9: 4.0, 5.1: 6.0, 7.0: 6.0, 100.0: 6.0}.items():
        assert orc.e2m1_decode(orc.e2m1_encode(x)) == want


def test_fp4_group_scale_closed_form(orc):
    assert orc.fp4_group_scale(0.0) == 1.0
    for e in range(-20, 20):
        edge = 6.0 * 2.0 ** e
        assert orc.fp4_group_scale(edge) == 2.0 ** e                 # amax = 6 sigma exactly
        assert orc.fp4_group_scale(math.nextafter(edge, math.inf)) == 2.0 ** (e + 1)
        assert orc.fp4_group_scale(math.nextafter(edge, 0.0)) == 2.0 ** e
    assert orc.fp4_group_scale(1e-3) == 2.0 ** -12
    assert orc.fp4_group_scale(3.0) == 0.5


def test_fp4_quantize_pack_order_and_error(orc):
    rng = np.random.default_rng(3)
    for _ in range(50):
        u = rng.standard_normal(64) * 10.0 ** rng.uniform(-3, 3)
        codes, scales = orc.fp4_quantize64(u)
        back = orc.fp4_dequantize64(codes, scales)
        for gi in range(2):
            grp = slice(32 * gi, 32 * gi + 32)
            amax = np.abs(u[grp]).max()
            s = float(scales[gi])
            assert amax <= 6 * s and amax > 3 * s                   # smallest fitting power of two
            # the error is at most half the local grid spacing (spacing <= 2*s)
            assert np.all(np.abs(back[grp] - u[grp]) <= s + 1e-12)
        # element 0 sits in the low nibble of byte 0, element 1 in the high nibble
        assert orc.e2m1_decode(codes[0] & 0xF) * scales[0] == back[0]
        assert orc.e2m1_decode(codes[0] >> 4) * scales[0] == back[1]


def test_entry_layout(orc):
    x = np.zeros(512)
    x[0], x[447], x[448], x[511] = 1.0, -2.0, 3.0, -0.5
    e = orc.entry_encode(x)
    assert e.shape == (576,)
    assert e[0] == 0x38 and e[447] == 0xC0                           # E4M3 1.0 and -2.0
    assert int(e[448]) | (int(e[449]) << 8) == 0x4040                          # bf16 3.0, little-endian
    assert int(e[574]) | (int(e[575]) << 8) == 0xBF00                          # bf16 -0.5
    assert np.array_equal(orc.entry_decode(e), x)


# ------------------------------------------------------------------------------------------
# O1 pooling: closed forms and invariants.
# ------------------------------------------------------------------------------------------
def _bf16_rows(m, seed):
    g = torch.Generator().manual_seed(seed)
    rows = torch.randn((m, 512), generator=g).to(torch.bfloat16)
    return synth.bits16(rows), rows.to(torch.float64).numpy()


@pytest.mark.parametrize("m", [1, 2, 4, 128])
def test_pool_constant_gates_is_mean(orc, m):
    bits, rows = _bf16_rows(m, 10 + m)
    gate = np.full(m, 0.7, np.float32)
    c = orc.pool_block(bits, gate, np.zeros(m, np.float32))
    assert np.allclose(c, rows.mean(axis=0), rtol=0, atol=1e-12)


def test_pool_two_token_closed_form(orc):
    bits, rows = _bf16_rows(2, 11)
    z = np.array([0.3, -1.1], np.float32)
    b = np.array([0.05, -0.2], np.float32)
    a = z.astype(np.float64) + b.astype(np.float64)
    w0 = 1.0 / (1.0 + math.exp(a[1] - a[0]))                       # sigmoid of the logit gap
    c = orc.pool_block(bits, z, b)
    assert np.allclose(c, w0 * rows[0] + (1 - w0) * rows[1], rtol=0, atol=1e-12)


def test_pool_dominant_logit_and_bias_slot(orc):
    bits, rows = _bf16_rows(4, 12)
    for j in range(4):
        z = np.zeros(4, np.float32)
        z[j] = 60.0
        assert np.allclose(orc.pool_block(bits, z, np.zeros(4, np.float32)), rows[j], rtol=1e-12, atol=1e-20)
        # the positional bias is indexed by the slot inside the block
        b = np.full(4, -60.0, np.float32)
        b[j] = 0.0
        assert np.allclose(orc.pool_block(bits, np.zeros(4, np.float32), b), rows[j], rtol=1e-12, atol=1e-20)


def test_pool_shift_invariance_and_softmax_weights(orc):
    bits, rows = _bf16_rows(128, 13)
    rng = np.random.default_rng(4)
    # logits on a 2^-10 grid, so that adding 3 is exact in fp32
    z = (np.round(rng.standard_normal(128) * 1024) / 1024).astype(np.float32)
    b = (rng.standard_normal(128) * 0.1).astype(np.float32)
    c1 = orc.pool_block(bits, z, b)
    c2 = orc.pool_block(bits, (z + np.float32(3.0)).astype(np.float32), b)
    assert np.allclose(c1, c2, rtol=0, atol=1e-12)
    w = torch.softmax(torch.from_numpy(z.astype(np.float64) + b.astype(np.float64)), 0).numpy()
    assert np.allclose(c1, w @ rows, rtol=0, atol=1e-12)


def test_identical_tokens_give_that_token(orc):
    g = torch.Generator().manual_seed(14)
    tok = torch.randn(512, generator=g).to(torch.bfloat16)
    bits = np.tile(synth.bits16(tok), (4, 1))
    z = np.array([0.1, -2.0, 1.5, 0.3], np.float32)
    c = orc.pool_block(bits, z, np.array([0.01, 0.02, -0.03, 0.0], np.float32))
    e = orc.entry_encode(c)
    ref = orc.entry_encode(tok.to(torch.float64).numpy())
    ordg = np.where(e[:448] & 0x80, -(e[:448] & 0x7F).astype(int), (e[:448] & 0x7F).astype(int))
    ordr = np.where(ref[:448] & 0x80, -(ref[:448] & 0x7F).astype(int), (ref[:448] & 0x7F).astype(int))
    assert np.abs(ordg - ordr).max() <= 1
    rg = e[448:].view(np.uint16).astype(int)
    rr = ref[448:].view(np.uint16).astype(int)
    assert np.abs(rg - rr).max() <= 1


# ------------------------------------------------------------------------------------------
# O2 indexer key: linearity (pool-then-project == project-then-pool).
# ------------------------------------------------------------------------------------------
def test_indexer_key_linearity(orc):
    bits, rows = _bf16_rows(4, 15)
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((512, 64)) / math.sqrt(512)).astype(np.float32)
    z = rng.standard_normal(4).astype(np.float32)
    b = (rng.standard_normal(4) * 0.1).astype(np.float32)
    u = orc.indexer_key_raw(orc.pool_block(bits, z, b), W)
    w = torch.softmax(torch.from_numpy(z.astype(np.float64) + b.astype(np.float64)), 0).numpy()
    per_token = rows @ W.astype(np.float64)
    assert np.allclose(u, w @ per_token, rtol=0, atol=1e-12)


def test_compress_matches_blockwise_pool(orc):
    inp = synth.prefill_inputs(4 * 9 + 3, seed=6)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    kv, ik, isc = orc.compress(bits, gate, inp["bias4"].numpy(), 4, inp["w_idx"].numpy())
    assert kv.shape == (9, 576) and ik.shape == (9, 32)                 # trailing 3 tokens: no entry
    for s in range(9):
        c = orc.pool_block(bits[4 * s:4 * s + 4], gate[4 * s:4 * s + 4], inp["bias4"].numpy())
        assert np.array_equal(kv[s], orc.entry_encode(c))
        codes, scales = orc.fp4_quantize64(orc.indexer_key_raw(c, inp["w_idx"].numpy()))
        assert np.array_equal(ik[s], codes) and np.array_equal(isc[s], scales)


# ------------------------------------------------------------------------------------------
# O3 indexer scores: exact rational arithmetic on tiny inputs.
# ------------------------------------------------------------------------------------------
def _exact_scores(orc, ikeys, iscales, q_idx, head_w, with_magnitude=False):
    qd = []
    for h in range(4):
        c, s = orc.fp4_quantize64(q_idx[h].astype(np.float64))
        qd.append([Fraction(v) for v in orc.fp4_dequantize64(c, s)])
    out, mag = [], []
    for n in range(ikeys.shape[0]):
        kd = [Fraction(v) for v in orc.fp4_dequantize64(ikeys[n], iscales[n])]
        e = Fraction(0)
        a = Fraction(0)
        for h in range(4):
            dot = sum(a_ * b_ for a_, b_ in zip(qd[h], kd))
            term = Fraction(float(head_w[h])) * max(dot, Fraction(0))
            e += term
            a += abs(term)
        out.append(e)
        mag.append(a)
    return (out, mag) if with_magnitude else out


def test_indexer_scores_exact(orc):
    g = synth.gen(7)
    ik, isc = synth.random_ikeys(1, 64, g, heavy_frac=0.1)
    ik, isc = ik[0].numpy(), isc[0].numpy()
    rng = np.random.default_rng(8)
    q = rng.standard_normal((4, 64)).astype(np.float32)
    w = np.abs(rng.standard_normal(4)).astype(np.float32)
    w[2] = -w[2]                                                       # a negative head weight
    s32, s64 = orc.indexer_scores(ik, isc, q, w)
    exact, mag = _exact_scores(orc, ik, isc, q, w, with_magnitude=True)
    for n in range(64):
        assert abs(Fraction(s64[n]) - exact[n]) <= mag[n] * Fraction(1, 10 ** 14)
        # fp32 score: 4 roundings, each at most 2^-24 of an intermediate bounded by sum |w_h r_h|
        assert abs(Fraction(float(s32[n])) - exact[n]) <= 4 * mag[n] / 2 ** 24


def test_indexer_single_head_dot_is_exact_in_fp32(orc):
    g = synth.gen(9)
    ik, isc = synth.random_ikeys(1, 200, g, heavy_frac=0.05)
    ik, isc = ik[0].numpy(), isc[0].numpy()
    rng = np.random.default_rng(10)
    q = rng.standard_normal((4, 64)).astype(np.float32)
    for h in range(4):
        w = np.zeros(4, np.float32)
        w[h] = 1.0
        s32, _ = orc.indexer_scores(ik, isc, q, w)
        exact = _exact_scores(orc, ik, isc, q, w)
        assert all(Fraction(float(a)) == b for a, b in zip(s32, exact))


def test_indexer_relu_drops_negative_dots(orc):
    q = np.zeros((4, 64), np.float32)
    q[:, 0] = 1.0                                                      # every head looks at dim 0
    codes = np.zeros((2, 32), np.uint8)
    codes[0, 0] = 0x0A                                                 # dim 0 = -1 (code 1010)
    codes[1, 0] = 0x02                                                 # dim 0 = +1
    sc = np.ones((2, 2), np.float32)
    s32, s64 = orc.indexer_scores(codes, sc, q, np.ones(4, np.float32))
    assert s32[0] == 0.0 and s64[0] == 0.0
    assert s32[1] == 4.0 and s64[1] == 4.0


# ------------------------------------------------------------------------------------------
# O4 top-k: brute force with many exact ties.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(0, 4), (3, 8), (50, 7), (200, 64), (257, 256)])
def test_topk_bruteforce(orc, n, k):
    rng = np.random.default_rng(n * 31 + k)
    s = rng.integers(0, 6, n).astype(np.float32) * np.float32(0.25)     # heavy ties
    got = orc.topk(s, k)
    order = sorted(range(n), key=lambda i: (-float(s[i]), i))[:k]
    want = sorted(order) + [-1] * (k - min(n, k))
    assert got.tolist() == want


def test_topk_union_of_chunk_topk_is_global(orc):
    rng = np.random.default_rng(11)
    s = rng.integers(0, 40, 1000).astype(np.float32)
    k = 37
    cands = []
    for c0 in range(0, 1000, 128):
        part = orc.topk(s[c0:c0 + 128], k)
        cands += [c0 + int(i) for i in part if i >= 0]
    sub = orc.topk(s[cands], k)
    merged = sorted(cands[int(i)] for i in sub if i >= 0)
    assert merged == orc.topk(s, k).tolist()


# ------------------------------------------------------------------------------------------
# O5 attention: brute force with a library softmax, special cases and invariants.
# ------------------------------------------------------------------------------------------
def _torch_attention(q64, keys64, scale):
    """Textbook softmax attention in float64 via torch (keys are also the values)."""
    if keys64.shape[0] == 0:
        return np.zeros_like(q64), np.full(q64.shape[0], -np.inf)
    qt = torch.from_numpy(q64)
    kt = torch.from_numpy(keys64)
    logits = scale * (qt @ kt.T)
    return (torch.softmax(logits, -1) @ kt).numpy(), torch.logsumexp(logits, -1).numpy()


def _case(orc, n, m, W, H=4, seed=0, cap=None):
    inp = synth.prefill_inputs(n, seed=seed)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"].numpy()[:1].repeat(m) if m != 4 else inp["bias4"].numpy()
    kv, _, _ = orc.compress(bits, gate, bias.astype(np.float32), m)
    cap = cap if cap is not None else max(1, kv.shape[0])
    comp = np.zeros((1, cap, 576), np.uint8)
    comp[0, :kv.shape[0]] = kv
    win = np.zeros((1, max(W, 0), 576), np.uint8)
    for t in range(max(0, n - W), n):
        win[0, t % W] = orc.entry_encode(inp["raw"][t].to(torch.float64).numpy())
    q = synth.decode_queries(1, seed=seed + 1, heads=H)["q"]
    return dict(bits=bits, raw=inp["raw"], comp=comp, kv=kv, win=win, q=q,
                qbits=synth.bits16(q), q64=q[0].to(torch.float64).numpy())


def test_identity_pooling_full_attention(orc):
    """m = 1, all entries selected, no window: exactly softmax attention over all n tokens."""
    n = 37
    cs = _case(orc, n, m=1, W=0)
    keys = orc.entries_decode(cs["kv"])
    ref_o, ref_l = _torch_attention(cs["q64"], keys, 0.05)
    sel = np.arange(n, dtype=np.int32)[None]
    for s in (None, sel):
        o, l = orc.attention_batch(cs["qbits"], cs["comp"], 1, s, cs["win"], np.array([n], np.int32), 0.05)
        assert np.allclose(o[0], ref_o, rtol=0, atol=1e-12) and np.allclose(l[0], ref_l, atol=1e-12)


def test_window_branch_bruteforce(orc):
    n, W, m = 45, 16, 4
    cs = _case(orc, n, m=m, W=W)
    raw64 = cs["raw"].to(torch.float64).numpy()
    win_keys = np.stack([orc.entry_decode(orc.entry_encode(raw64[t])) for t in range(n - W, n)])
    keys = np.concatenate([orc.entries_decode(cs["kv"]), win_keys])
    ref_o, ref_l = _torch_attention(cs["q64"], keys, 0.07)
    o, l = orc.attention_batch(cs["qbits"], cs["comp"], m, None, cs["win"], np.array([n], np.int32), 0.07)
    assert np.allclose(o[0], ref_o, atol=1e-12) and np.allclose(l[0], ref_l, atol=1e-12)


def test_topk_covering_all_entries_equals_dense(orc):
    n, W, m = 64, 8, 4
    cs = _case(orc, n, m=m, W=W)
    sel = np.array([list(range(16)) + [-1] * 4], np.int32)                 # k = 20 >= 16 entries
    od, ld = orc.attention_batch(cs["qbits"], cs["comp"], m, None, cs["win"], np.array([n], np.int32), 0.04)
    os_, ls = orc.attention_batch(cs["qbits"], cs["comp"], m, sel, cs["win"], np.array([n], np.int32), 0.04)
    assert np.allclose(od, os_, atol=1e-13) and np.allclose(ld, ls, atol=1e-13)


def test_permutation_and_lse_merge(orc):
    n, m = 80, 4
    cs = _case(orc, n, m=m, W=0)
    scale = 0.06
    sl = np.array([n], np.int32)
    a = np.array([[3, 7, 0, 19, 11]], np.int32)
    b = np.array([[1, 2, 4, 5, 6, 8, 9, 10]], np.int32)
    ab = np.concatenate([a, b], 1)
    o1, l1 = orc.attention_batch(cs["qbits"], cs["comp"], m, ab, cs["win"], sl, scale)
    o2, l2 = orc.attention_batch(cs["qbits"], cs["comp"], m, ab[:, ::-1].copy(), cs["win"], sl, scale)
    assert np.allclose(o1, o2, atol=1e-13)
    oa, la = orc.attention_batch(cs["qbits"], cs["comp"], m, a, cs["win"], sl, scale)
    ob, lb = orc.attention_batch(cs["qbits"], cs["comp"], m, b, cs["win"], sl, scale)
    lm = np.logaddexp(la, lb)
    om = (np.exp(la - lm)[..., None] * oa + np.exp(lb - lm)[..., None] * ob)
    assert np.allclose(om, o1, atol=1e-12) and np.allclose(lm, l1, atol=1e-12)


def test_short_sequence_is_window_only(orc):
    n, W, m = 3, 8, 4                                                      # n < m: nothing compressed
    cs = _case(orc, n, m=m, W=W, cap=4)
    raw64 = cs["raw"].to(torch.float64).numpy()
    keys = np.stack([orc.entry_decode(orc.entry_encode(raw64[t])) for t in range(n)])
    ref_o, ref_l = _torch_attention(cs["q64"], keys, 0.05)
    o, l = orc.attention_batch(cs["qbits"], cs["comp"], m, None, cs["win"], np.array([n], np.int32), 0.05)
    assert np.allclose(o[0], ref_o, atol=1e-12) and np.allclose(l[0], ref_l, atol=1e-12)
    o0, l0 = orc.attention_batch(cs["qbits"], cs["comp"], m, None, cs["win"], np.array([0], np.int32), 0.05)
    assert np.all(o0 == 0) and np.all(np.isneginf(l0))


def test_attention_rejects_invisible_index(orc):
    cs = _case(orc, 16, m=4, W=4)
    with pytest.raises(ValueError):
        orc.attention_batch(cs["qbits"], cs["comp"], 4, np.array([[0, 4]], np.int32), cs["win"],
                            np.array([16], np.int32), 0.05)


# ------------------------------------------------------------------------------------------
# O6 append: token-by-token append reproduces prefill compression; capacity is enforced.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("m,W,idx", [(4, 16, True), (128, 32, False), (1, 4, False)])
def test_append_equals_prefill(orc, m, W, idx):
    T = 2 * 128 + 37
    inp = synth.prefill_inputs(T, seed=20)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"].numpy() if m == 4 else (inp["bias128"].numpy() if m == 128 else np.zeros(1, np.float32))
    w_idx = inp["w_idx"].numpy() if idx else None
    kv, ik, isc = orc.compress(bits, gate, bias, m, w_idx)
    E = T // m
    st = orc.LayerState(1, E + 1, m, W, idx)
    for t in range(T):
        orc.append_batch(st, bias, w_idx, bits[t:t + 1], gate[t:t + 1])
    assert st.seq_len[0] == T
    assert np.array_equal(st.comp_kv[0, :E], kv)
    if idx:
        assert np.array_equal(st.ikeys[0, :E], ik) and np.array_equal(st.iscales[0, :E], isc)
    raw64 = inp["raw"].to(torch.float64).numpy()
    for t in range(T - W, T):
        assert np.array_equal(st.win_kv[0, t % W], orc.entry_encode(raw64[t]))
    for t in range(T - T % m, T):
        assert np.array_equal(st.tail_kv[0, t % m], bits[t]) and st.tail_gate[0, t % m] == gate[t]


def test_append_capacity_overflow_changes_nothing(orc):
    inp = synth.prefill_inputs(8, seed=21)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    st = orc.LayerState(1, 1, 4, 4, False)
    for t in range(7):
        orc.append_batch(st, inp["bias4"].numpy(), None, bits[t:t + 1], gate[t:t + 1])
    before = (st.win_kv.copy(), st.tail_kv.copy(), st.seq_len.copy())
    with pytest.raises(OverflowError):
        orc.append_batch(st, inp["bias4"].numpy(), None, bits[7:8], gate[7:8])
    assert np.array_equal(before[0], st.win_kv) and np.array_equal(before[1], st.tail_kv)
    assert np.array_equal(before[2], st.seq_len)


# ------------------------------------------------------------------------------------------
# Byte accounting against the pages' figures (ratios, "about 2%" of a GQA-8 bf16 cache).
# ------------------------------------------------------------------------------------------
def test_kv_byte_accounting_reproduces_page_figure(orc):
    fig = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
    r_csa, r_hca = fig["csa_ratio"]["value"], fig["hca_ratio"]["value"]
    lp = fig["layer_pattern"]["value"]
    # entry sizes measured from the oracle's own encoders
    entry = orc.entry_encode(np.zeros(512)).nbytes
    codes, scales = orc.fp4_quantize64(np.zeros(64))
    ikey = codes.nbytes + scales.nbytes
    assert (entry, ikey) == (576, 40)
    kinds = ["HCA" if l in lp["hca_only"] else ("CSA" if (l - lp["alternating"][0]) % 2 == 0 else "HCA")
             for l in range(lp["layers"])]
    n_csa, n_hca = kinds.count("CSA"), kinds.count("HCA")
    assert (n_csa, n_hca) == (30, 31)
    per_token = n_csa * (entry + ikey) / r_csa + n_hca * entry / r_hca
    gqa8 = lp["layers"] * 8 * 128 * 2 * 2                                 # 8 KV heads, dim 128, K and V, bf16
    frac = per_token / gqa8
    assert abs(frac - fig["kv_fraction_vs_gqa8_bf16"]["value"]) < 0.005, frac
    # entry counts of the 4096-token case
    assert 4096 // r_csa == 1024 and 4096 // r_hca == 32


# ---- per-channel gating (layout / gating variant) ---------------------------------------------
def test_pool_channel_reduces_to_scalar_gating(orc):
    """Gates and biases equal across dimensions: per-channel pooling is the scalar pooling."""
    rng = np.random.default_rng(5)
    for m in (1, 4, 7, 128):
        raw = rng.standard_normal((m, 512)).astype(np.float32)
        bits = (raw.view(np.uint32) >> 16).astype(np.uint16)
        z = rng.standard_normal(m).astype(np.float32)
        b = (0.1 * rng.standard_normal(m)).astype(np.float32)
        ref = orc.pool_block(bits, z, b)
        got = orc.pool_block_channel(bits, np.repeat(z[:, None], 512, 1), np.repeat(b[:, None], 512, 1))
        assert np.allclose(got, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))


def test_pool_channel_dims_are_independent(orc):
    """A dominant logit on one dimension picks that slot's value there; a dimension with equal
    logits is the mean; the other dimensions do not see either."""
    m = 4
    rng = np.random.default_rng(6)
    raw = rng.standard_normal((m, 512)).astype(np.float32)
    bits = (raw.view(np.uint32) >> 16).astype(np.uint16)
    x = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    gate = np.zeros((m, 512), np.float32)
    bias = np.zeros((m, 512), np.float32)
    gate[2, 10] = 80.0                      # dim 10: slot 2 dominates
    gate[:, 11] = rng.standard_normal(m)     # dim 11: a softmax of its own
    c = orc.pool_block_channel(bits, gate, bias)
    assert abs(c[10] - x[2, 10]) < 1e-12
    w = np.exp(gate[:, 11].astype(np.float64) - gate[:, 11].max())
    w /= w.sum()
    assert abs(c[11] - (w * x[:, 11]).sum()) < 1e-12
    others = [d for d in range(512) if d not in (10, 11)]
    assert np.allclose(c[others], x[:, others].mean(0), rtol=0, atol=1e-12)


def test_compress_channel_shift_invariance(orc):
    """Adding a constant to one dimension's logits of a block leaves the entry unchanged."""
    m, T = 4, 64
    rng = np.random.default_rng(7)
    raw = rng.standard_normal((T, 512)).astype(np.float32)
    bits = (raw.view(np.uint32) >> 16).astype(np.uint16)
    gate = rng.standard_normal((T, 512)).astype(np.float32)
    bias = (0.1 * rng.standard_normal((m, 512))).astype(np.float32)
    kv0, _, _ = orc.compress_channel(bits, gate, bias, m)
    g2 = gate.copy()
    g2[4:8, 100] += 3.0                     # block 1, dimension 100
    kv1, _, _ = orc.compress_channel(bits, g2, bias, m)
    assert np.array_equal(kv0, kv1)
