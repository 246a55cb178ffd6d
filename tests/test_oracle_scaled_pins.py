"""Pins of the oracle's scaled-FP8-entry variant (no GPU needed).

One positive scale sigma per layer cache: an entry's E4M3 dims hold E4M3(x / sigma) and stand
for sigma times their code value; the bf16 RoPE dims are not scaled.  The pins tie it to the
base layout (sigma = 1), to exact power-of-two scaling of E4M3 values, to saturation at
448 sigma, to attention computed by torch in float64 over the decoded entries, and to the base
reading's append = prefill.
"""
import numpy as np
import pytest
import torch

import synth


def _e4m3_grid(orc):
    return np.array([orc.e4m3_decode(c) for c in range(256) if (c & 0x7F) != 0x7F])


def test_unit_scale_is_the_base_layout(orc):
    rng = np.random.default_rng(11)
    x = rng.standard_normal(512) * 3
    assert np.array_equal(orc.entry_encode_scaled(x, 1.0), orc.entry_encode(x))
    inp = synth.prefill_inputs(4 * 50 + 1, seed=41)
    bits = synth.bits16(inp["raw"])
    a = orc.compress(bits, inp["gate"].numpy(), inp["bias4"].numpy(), 4, inp["w_idx"].numpy())
    b = orc.compress_scaled(bits, inp["gate"].numpy(), inp["bias4"].numpy(), 4, 1.0, inp["w_idx"].numpy())
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("k", [-6, -1, 3])
def test_power_of_two_scale_is_exact_on_e4m3_values(orc, k):
    """x = 2^k * (an E4M3 value in the normal range) encodes to that value's code and decodes
    back to x exactly: the scale divides before rounding and multiplies after decoding."""
    grid = _e4m3_grid(orc)
    normal = grid[(np.abs(grid) >= 2.0 ** -6) & (np.abs(grid) <= 448)]
    rng = np.random.default_rng(12 + k)
    vals = rng.choice(normal, 448)
    x = np.concatenate([vals * 2.0 ** k, rng.standard_normal(64)])
    e = orc.entry_encode_scaled(x, 2.0 ** k)
    assert np.array_equal(e[:448], orc.entry_encode(np.concatenate([vals, x[448:]]))[:448])
    back = orc.entry_decode_scaled(e, 2.0 ** k)
    assert np.array_equal(back[:448], x[:448])
    assert np.array_equal(e[448:], orc.entry_encode(x)[448:])       # RoPE dims untouched


def test_saturation_at_448_sigma(orc):
    sigma = 0.37
    x = np.zeros(512)
    x[0], x[1], x[2] = 1e6, -1e6, 448 * sigma * 0.999
    back = orc.entry_decode_scaled(orc.entry_encode_scaled(x, sigma), sigma)
    assert back[0] == pytest.approx(448 * sigma, rel=1e-15) and back[1] == pytest.approx(-448 * sigma, rel=1e-15)
    assert abs(back[2] - x[2]) <= 2.0 ** -4 * abs(x[2])


def test_scale_widens_the_range_of_small_values(orc):
    """Values far below E4M3's smallest subnormal (2^-9) vanish unscaled and survive a small
    sigma within E4M3's relative precision."""
    x = np.zeros(512)
    x[:448] = np.linspace(1e-5, 4e-4, 448)
    assert not orc.entry_decode(orc.entry_encode(x))[:448][:10].any()
    sigma = 4e-4 / 448
    back = orc.entry_decode_scaled(orc.entry_encode_scaled(x, sigma), sigma)
    assert np.all(np.abs(back[:448] - x[:448]) <= 2.0 ** -4 * x[:448] + 1e-30)


def test_scaled_attention_matches_torch_over_decoded_entries(orc):
    """Attention over scaled entries equals float64 softmax attention (torch) over the entries'
    decoded values, E4M3 dims times sigma."""
    rng = np.random.default_rng(13)
    B, cap, W, n, sigma = 2, 40, 8, 4 * 40, 0.0123
    comp = rng.integers(0, 256, (B, cap, 576), dtype=np.uint8)
    comp[:, :, :448] &= 0xF7                       # finite E4M3 codes of both signs (exponent < 15)
    comp[:, :, 448:] = 0
    win = comp[:, :W].copy()
    q = (rng.standard_normal((B, 16, 512)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    seq = np.full(B, n, np.int32)
    scale = 0.05
    out, lse = orc.attention_batch(q, comp, 4, None, win, seq, scale, kv_scale=sigma)
    qd = torch.from_numpy((q.astype(np.uint32) << 16).view(np.float32)).double()
    for b in range(B):
        rows = [orc.entry_decode(comp[b, s]) for s in range(n // 4)]
        rows += [orc.entry_decode(win[b, t % W]) for t in range(n - W, n)]
        kv = torch.tensor(np.array(rows))
        kv[:, :448] *= sigma
        logits = scale * qd[b] @ kv.T
        ref = torch.softmax(logits, -1) @ kv
        assert torch.allclose(torch.from_numpy(out[b]), ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse[b], torch.logsumexp(logits, -1).numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("m,W,idx", [(4, 16, True), (128, 32, False)])
def test_append_scaled_equals_prefill_scaled(orc, m, W, idx):
    T = 2 * 128 + 37
    inp = synth.prefill_inputs(T, seed=42)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"].numpy() if m == 4 else inp["bias128"].numpy()
    w_idx = inp["w_idx"].numpy() if idx else None
    sigma = 0.0071
    kv, ik, isc = orc.compress_scaled(bits, gate, bias, m, sigma, w_idx)
    kv0, ik0, isc0 = orc.compress(bits, gate, bias, m, w_idx)
    assert not np.array_equal(kv[:, :448], kv0[:, :448]) and np.array_equal(kv[:, 448:], kv0[:, 448:])
    if idx:   # the key comes from the unscaled pooled vector
        assert np.array_equal(ik, ik0) and np.array_equal(isc, isc0)
    E = T // m
    st = orc.LayerState(1, E + 1, m, W, idx)
    for t in range(T):
        orc.append_batch(st, bias, w_idx, bits[t:t + 1], gate[t:t + 1], kv_scale=sigma)
    assert np.array_equal(st.comp_kv[0, :E], kv)
    raw64 = inp["raw"].to(torch.float64).numpy()
    for t in range(T - W, T):
        assert np.array_equal(st.win_kv[0, t % W], orc.entry_encode_scaled(raw64[t], sigma))
