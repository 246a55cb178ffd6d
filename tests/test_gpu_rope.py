"""GPU parity of the RoPE-at-compressed-positions variant (csld_compress_rope,
kv_cache_prefill_rope, kv_cache_append_rope) against the float64 oracle on the same seeded
inputs: entry bytes (E4M3 codes within one step, bf16 RoPE dims within one bf16 step plus the
pooling's fp32 slack, doubled because a rotation mixes two pooled dims), FP4 keys, window
ring, tail and lengths."""
import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu
BASE = 10000.0


@pytest.fixture(scope="module")
def csld():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_long_decode_b200 as m
    return m


def _rope_ramax(orc, bits, gate, bias, m, w_idx, positions):
    """Per-group max |u| of the oracle's unquantised keys of the rotated vectors."""
    out = np.zeros((len(positions), 2))
    for s, p in enumerate(positions):
        c = orc.rope_rotate(orc.pool_block(bits[s * m:(s + 1) * m], gate[s * m:(s + 1) * m], bias), p, BASE)
        u = orc.indexer_key_raw(c, w_idx)
        out[s] = [np.abs(u[:32]).max(), np.abs(u[32:]).max()]
    return out


@pytest.mark.parametrize("T,m,idx,pos0", [(4096 + 37, 4, True, 0), (2048 + 5, 4, True, 3_000_000),
                                          (128 * 33 + 17, 128, False, 1_000_000), (501, 7, False, 12345),
                                          (300, 1, False, 7)])
def test_compress_rope_matches_oracle(csld, orc, T, m, idx, pos0):
    inp = synth.prefill_inputs(T, seed=900 + T + m)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    if m == 4:
        bias = inp["bias4"]
    elif m == 128:
        bias = inp["bias128"]
    else:
        bias = torch.randn(m, generator=synth.gen(m), dtype=torch.float32) * 0.1
    w = inp["w_idx"] if idx else None
    got = csld.compress_rope(inp["raw"].cuda(), inp["gate"].cuda(), bias.cuda(), m, pos0, BASE,
                             None if w is None else w.cuda())
    torch.cuda.synchronize()
    rkv, rik, risc = orc.compress_rope(bits, gate, bias.numpy(), m, pos0, BASE, None if w is None else w.numpy())
    kv = (got[0] if idx else got).cpu().numpy()
    slack = 2 * H.pool_slack(inp["raw"], m) + 2.0 ** -23 * float(inp["raw"].float().abs().max())
    frac = H.assert_entries_close(kv, rkv, f"ratio-{m} RoPE entries", slack)
    assert frac > 0.99
    if idx:
        ik, isc = got[1].cpu().numpy(), got[2].cpu().numpy()
        positions = [pos0 + (s + 1) * m - 1 for s in range(T // m)]
        ramax = None if np.array_equal(isc, risc) else _rope_ramax(orc, bits, gate, bias.numpy(), m, w.numpy(),
                                                                   positions)
        H.assert_fp4_keys_close(synth.ikeys_swap_halves(ik), isc, rik, risc, ramax)


def test_compress_rope_differs_from_base_only_in_rope_dims(csld):
    """The E4M3 dims of the variant's entries are the base compressor's bytes exactly."""
    T = 4 * 300
    inp = synth.prefill_inputs(T, seed=951)
    raw, gate, bias = inp["raw"].cuda(), inp["gate"].cuda(), inp["bias4"].cuda()
    base = csld.compress(raw, gate, bias, 4).cpu().numpy()
    rope = csld.compress_rope(raw, gate, bias, 4, 100, BASE).cpu().numpy()
    assert np.array_equal(base[:, :448], rope[:, :448])
    assert not np.array_equal(base[:, 448:], rope[:, 448:])


def _window_close(win, win_ref, seq_len, W):
    for b, n in enumerate(np.asarray(seq_len).tolist()):
        for t in range(max(0, n - W), n):
            g, r = win[b, t % W], win_ref[b, t % W]
            assert np.array_equal(g[:448], r[:448]), f"window E4M3 bytes of token {t}"
            gv = H.bf16_values(g[448:].copy().view(np.uint16))
            rv = H.bf16_values(r[448:].copy().view(np.uint16))
            assert np.all(np.abs(gv - rv) <= H.bf16_ulp(rv)), f"window RoPE dims of token {t}"


@pytest.mark.parametrize("m,W,idx,T,steps", [(4, 128, True, 1021, 23), (128, 64, False, 128 * 5 + 100, 40)])
def test_prefill_and_append_rope_match_oracle(csld, orc, m, W, idx, T, steps):
    B = 3
    parts = [synth.prefill_inputs(T + steps, seed=960 + 7 * b_ + m) for b_ in range(B)]
    raw = torch.stack([p["raw"] for p in parts])
    gate = torch.stack([p["gate"] for p in parts])
    bias = parts[0]["bias4"] if m == 4 else parts[0]["bias128"]
    w_idx = parts[0]["w_idx"] if idx else None
    cap = (T + steps) // m + 2
    cache = csld.LayerCache(B, cap, m, W, bias, w_idx)
    csld.kv_cache_prefill_rope(cache, raw[:, :T].contiguous().cuda(), gate[:, :T].contiguous().cuda(), BASE)
    for t in range(T, T + steps):
        csld.kv_cache_append_rope(cache, raw[:, t].contiguous().cuda(), gate[:, t].contiguous().cuda(), BASE)
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    bits = raw.view(torch.int16).numpy().view(np.uint16)
    g = gate.numpy()
    st = orc.LayerState(B, cache.capacity, m, W, idx)
    for t in range(T + steps):
        orc.append_batch(st, bias.numpy(), None if w_idx is None else w_idx.numpy(), bits[:, t].copy(),
                         g[:, t].copy(), rope_base=BASE)
    assert np.array_equal(cache.seq_len.cpu().numpy(), st.seq_len)
    n = (T + steps) // m
    slack = 2 * H.pool_slack(raw, m) + 2.0 ** -23 * float(raw.float().abs().max())
    H.assert_entries_close(cache.comp_kv[:, :n].cpu().numpy(), st.comp_kv[:, :n], "RoPE cache entries", slack)
    _window_close(cache.win_kv.cpu().numpy(), st.win_kv, st.seq_len, W)
    tail = cache.tail_kv.view(torch.int16).cpu().numpy().view(np.uint16)
    for b_ in range(B):
        for j in range((T + steps) % m):
            assert np.array_equal(tail[b_, j], st.tail_kv[b_, j]), "the tail keeps the tokens as given"
    if idx:
        for b_ in range(B):
            gs = cache.iscales[b_, :n].cpu().numpy()
            ramax = None
            if not np.array_equal(gs, st.iscales[b_, :n]):
                ramax = _rope_ramax(orc, bits[b_], g[b_], bias.numpy(), m, w_idx.numpy(),
                                    [(s + 1) * m - 1 for s in range(n)])
            H.assert_fp4_keys_close(synth.ikeys_swap_halves(cache.ikeys[b_, :n].cpu().numpy()), gs,
                                    st.ikeys[b_, :n], st.iscales[b_, :n], ramax)


def test_rope_entry_points_reject_bad_arguments(csld):
    inp = synth.prefill_inputs(16, seed=970)
    with pytest.raises(csld.CsldError):
        csld.compress_rope(inp["raw"].cuda(), inp["gate"].cuda(), inp["bias4"].cuda(), 4, 0, 0.5)
    with pytest.raises(csld.CsldError):
        csld.compress_rope(inp["raw"].cuda(), inp["gate"].cuda(), inp["bias4"].cuda(), 4, -1, BASE)
    cache = csld.LayerCache(1, 8, 4, 4, inp["bias4"])
    with pytest.raises(csld.CsldError):
        csld.kv_cache_append_rope(cache, inp["raw"][:1].contiguous().cuda(), inp["gate"][:1].contiguous().cuda(),
                                  float("inf"))
