"""GPU parity of the scaled-FP8-entry variant (csld_compress_scaled, kv_cache_prefill_scaled,
kv_cache_append_scaled, hybrid_decode_attention_scaled) against the float64 oracle on the same
seeded inputs: entry bytes (E4M3 codes within one step -- the device multiplies by 1 / sigma in
fp32 -- and bf16 RoPE dims within one bf16 step plus the pooling's fp32 slack), FP4 keys,
window ring, and attention within the usual bound."""
import math

import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(512.0)


@pytest.fixture(scope="module")
def csld():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_long_decode_b200 as m
    return m


def _ramax(orc, bits, gate, bias, m, w_idx, n):
    """Per-group max |u| of the oracle's unquantised keys (for the FP4 scale exemption)."""
    out = np.zeros((n, 2))
    for s in range(n):
        u = orc.indexer_key_raw(orc.pool_block(bits[s * m:(s + 1) * m], gate[s * m:(s + 1) * m], bias), w_idx)
        out[s] = [np.abs(u[:32]).max(), np.abs(u[32:]).max()]
    return out


@pytest.mark.parametrize("T,m,idx,sigma", [(4096 + 37, 4, True, 0.0071), (4096, 4, True, 2.0 ** -5),
                                           (128 * 33 + 17, 128, False, 0.013), (501, 7, False, 3.5)])
def test_compress_scaled_matches_oracle(csld, orc, T, m, idx, sigma):
    inp = synth.prefill_inputs(T, seed=1200 + T + m)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    if m == 4:
        bias = inp["bias4"]
    elif m == 128:
        bias = inp["bias128"]
    else:
        bias = torch.randn(m, generator=synth.gen(m), dtype=torch.float32) * 0.1
    w = inp["w_idx"] if idx else None
    got = csld.compress_scaled(inp["raw"].cuda(), inp["gate"].cuda(), bias.cuda(), m, sigma,
                               None if w is None else w.cuda())
    torch.cuda.synchronize()
    rkv, rik, risc = orc.compress_scaled(bits, gate, bias.numpy(), m, sigma, None if w is None else w.numpy())
    kv = (got[0] if idx else got).cpu().numpy()
    frac = H.assert_entries_close(kv, rkv, f"ratio-{m} scaled entries", H.pool_slack(inp["raw"], m))
    assert frac > 0.98
    if idx:   # the keys are those of the base layout
        ik, isc = got[1].cpu().numpy(), got[2].cpu().numpy()
        base = csld.compress(inp["raw"].cuda(), inp["gate"].cuda(), bias.cuda(), m, w.cuda())
        assert np.array_equal(ik, base[1].cpu().numpy()) and np.array_equal(isc, base[2].cpu().numpy())
        ramax = None if np.array_equal(isc, risc) else _ramax(orc, bits, gate, bias.numpy(), m, w.numpy(), T // m)
        H.assert_fp4_keys_close(synth.ikeys_swap_halves(ik), isc, rik, risc, ramax)


@pytest.mark.parametrize("m,W,idx,T,steps", [(4, 128, True, 1021, 23), (128, 64, False, 128 * 5 + 100, 40)])
def test_prefill_and_append_scaled_match_oracle(csld, orc, m, W, idx, T, steps):
    B, sigma = 2, 0.0093
    parts = [synth.prefill_inputs(T + steps, seed=1300 + 7 * b_ + m) for b_ in range(B)]
    raw = torch.stack([p["raw"] for p in parts])
    gate = torch.stack([p["gate"] for p in parts])
    bias = parts[0]["bias4"] if m == 4 else parts[0]["bias128"]
    w_idx = parts[0]["w_idx"] if idx else None
    cap = (T + steps) // m + 2
    cache = csld.LayerCache(B, cap, m, W, bias, w_idx)
    csld.kv_cache_prefill_scaled(cache, raw[:, :T].contiguous().cuda(), gate[:, :T].contiguous().cuda(), sigma)
    for t in range(T, T + steps):
        csld.kv_cache_append_scaled(cache, raw[:, t].contiguous().cuda(), gate[:, t].contiguous().cuda(), sigma)
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    bits = raw.view(torch.int16).numpy().view(np.uint16)
    g = gate.numpy()
    st = orc.LayerState(B, cache.capacity, m, W, idx)
    for t in range(T + steps):
        orc.append_batch(st, bias.numpy(), None if w_idx is None else w_idx.numpy(), bits[:, t].copy(),
                         g[:, t].copy(), kv_scale=sigma)
    assert np.array_equal(cache.seq_len.cpu().numpy(), st.seq_len)
    n = (T + steps) // m
    H.assert_entries_close(cache.comp_kv[:, :n].cpu().numpy(), st.comp_kv[:, :n], "scaled cache entries",
                           H.pool_slack(raw, m))
    win = cache.win_kv.cpu().numpy()
    for b_ in range(B):
        live = [t % W for t in range(T + steps - W, T + steps)]
        H.assert_entries_close(win[b_, live], st.win_kv[b_, live], "scaled window entries")
    if idx:
        for b_ in range(B):
            gs = cache.iscales[b_, :n].cpu().numpy()
            ramax = None
            if not np.array_equal(gs, st.iscales[b_, :n]):
                ramax = _ramax(orc, bits[b_], g[b_], bias.numpy(), m, w_idx.numpy(), n)
            H.assert_fp4_keys_close(synth.ikeys_swap_halves(cache.ikeys[b_, :n].cpu().numpy()), gs,
                                    st.ikeys[b_, :n], st.iscales[b_, :n], ramax)


@pytest.mark.parametrize("B,n,W,ratio,k,sigma", [(3, 128 * 40 + 5, 128, 128, 0, 0.05), (2, 4 * 3000, 64, 4, 512, 0.02),
                                                 (4, 4 * 500, 128, 4, 256, 3.0), (8, 128 * 65, 128, 128, 0, 0.7)])
def test_attention_scaled_matches_oracle(csld, orc, B, n, W, ratio, k, sigma):
    cap = n // ratio + 8
    g = synth.gen(1400 + n + B)
    comp = synth.random_entries((B, cap), g)
    win = synth.random_entries((B, W), g)
    q = synth.decode_queries(B, seed=1401 + n)["q"]
    seq = torch.full((B,), n, dtype=torch.int32)
    sel = None
    if k:
        sel = torch.stack([torch.randperm(n // ratio, generator=g)[:k].sort().values for _ in range(B)]).to(torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = csld.hybrid_decode_attention_scaled(q.cuda(), comp.cuda(), ratio, None if sel is None else sel.cuda(),
                                                   win.cuda(), W, seq.cuda(), SCALE, sigma, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ro, rl = orc.attention_batch(synth.bits16(q), comp.numpy(), ratio, None if sel is None else sel.numpy(),
                                 win.numpy(), seq.numpy(), SCALE, kv_scale=sigma)
    H.assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, f"scaled attention sigma={sigma}")


def test_attention_unit_scale_is_the_base_call(csld):
    B, n, W = 2, 4 * 2000, 128
    g = synth.gen(1500)
    comp = synth.random_entries((B, n // 4 + 4), g).cuda()
    win = synth.random_entries((B, W), g).cuda()
    q = synth.decode_queries(B, seed=1501)["q"].cuda()
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    sel = torch.stack([torch.randperm(n // 4, generator=g)[:512].sort().values for _ in range(B)]).to(torch.int32).cuda()
    o1, l1 = csld.hybrid_decode_attention(q, comp, 4, sel, win, W, seq, SCALE)
    o2, l2 = csld.hybrid_decode_attention_scaled(q, comp, 4, sel, win, W, seq, SCALE, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_scaled_entry_points_reject_bad_scales(csld):
    inp = synth.prefill_inputs(16, seed=1600)
    for bad in (0.0, -1.0, float("inf"), float("nan"), 2.0 ** 70):
        with pytest.raises(csld.CsldError):
            csld.compress_scaled(inp["raw"].cuda(), inp["gate"].cuda(), inp["bias4"].cuda(), 4, bad)
