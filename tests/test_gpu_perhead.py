"""GPU parity of the per-head-indexer-key variant (csld_compress_perhead, kv_cache_prefill_perhead,
kv_cache_append_perhead, indexer_topk_perhead) against the float64 oracle on the same seeded
inputs: entries bit-exact with the base compressor, FP4 keys of every head (codes within one step
at equal scales, scales equal except at a power-of-two boundary), and selections bit-exact with
the oracle's fp32 recipe and equal to its float64 selection up to near-ties."""
import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csld():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_long_decode_b200 as m
    return m


def _unswizzle(stored):
    """Stored per-head keys [..., E, 128] (chunk c of entry s at chunk c ^ (s mod 8)) -> the plain
    [..., E, 4, 32] layout of the oracle."""
    st = np.asarray(stored, np.uint8)
    chunks = st.reshape(st.shape[:-1] + (8, 16))
    out = np.empty_like(chunks)
    for c in range(8):
        for r in range(8):
            out[..., r::8, c, :] = chunks[..., r::8, c ^ r, :]
    return out.reshape(st.shape[:-1] + (4, 32))


def _swizzle(plain):
    """Plain [..., E, 4, 32] -> the stored [..., E, 128] layout."""
    pl = np.asarray(plain, np.uint8)
    E = pl.shape[-3]
    chunks = pl.reshape(pl.shape[:-2] + (8, 16))
    out = np.empty_like(chunks)
    for c in range(8):
        for r in range(8):
            out[..., r::8, c ^ r, :] = chunks[..., r::8, c, :]
    return out.reshape(pl.shape[:-2] + (128,))


def _perhead_w(rng):
    return (rng.standard_normal((512, 4, 64)) / np.sqrt(512)).astype(np.float32)


def _ramax(orc, bits, gate, bias, m, w, n):
    out = np.zeros((n, 4, 2))
    for s in range(n):
        u = orc.indexer_key_raw_perhead(orc.pool_block(bits[s * m:(s + 1) * m], gate[s * m:(s + 1) * m], bias), w)
        out[s, :, 0] = np.abs(u[:, :32]).max(1)
        out[s, :, 1] = np.abs(u[:, 32:]).max(1)
    return out


def _keys_close(gkeys_plain, gscales, rkeys, rscales, ramax_fn):
    for h in range(4):
        gs, rs = gscales[:, h], rscales[:, h]
        ramax = None if np.array_equal(gs, rs) else ramax_fn()[:, h]
        H.assert_fp4_keys_close(gkeys_plain[:, h], gs, rkeys[:, h], rs, ramax)


def test_swizzle_helpers_roundtrip():
    rng = np.random.default_rng(0)
    x = rng.integers(0, 256, (3, 37, 4, 32), dtype=np.uint8)
    assert np.array_equal(_unswizzle(_swizzle(x)), x)


@pytest.mark.parametrize("T,m", [(4096 + 37, 4), (4 * 37 + 3, 4), (128 * 5 + 17, 128)])
def test_compress_perhead_matches_oracle(csld, orc, T, m):
    inp = synth.prefill_inputs(T, seed=2000 + T + m)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()
    bias = inp["bias4"] if m == 4 else inp["bias128"]
    w = _perhead_w(np.random.default_rng(2001 + T))
    kv, ik, isc = csld.compress_perhead(inp["raw"].cuda(), inp["gate"].cuda(), bias.cuda(), m, torch.from_numpy(w).cuda())
    base = csld.compress(inp["raw"].cuda(), inp["gate"].cuda(), bias.cuda(), m)
    torch.cuda.synchronize()
    assert torch.equal(kv, base)                         # the entries are the base compressor's
    rkv, rik, risc = orc.compress_perhead(bits, gate, bias.numpy(), m, w)
    E = T // m
    _keys_close(_unswizzle(ik.cpu().numpy()), isc.cpu().numpy(), rik, risc,
                lambda: _ramax(orc, bits, gate, bias.numpy(), m, w, E))


@pytest.mark.parametrize("T,steps", [(1021, 23), (4 * 300, 9)])
def test_prefill_and_append_perhead_match_oracle(csld, orc, T, steps):
    B, m, W = 2, 4, 64
    parts = [synth.prefill_inputs(T + steps, seed=2100 + 7 * b_) for b_ in range(B)]
    raw = torch.stack([p["raw"] for p in parts])
    gate = torch.stack([p["gate"] for p in parts])
    bias = parts[0]["bias4"]
    w = _perhead_w(np.random.default_rng(2101 + T))
    cap = (T + steps) // m + 2
    cache = csld.LayerCache(B, cap, m, W, bias, torch.from_numpy(w), perhead=True)
    csld.kv_cache_prefill_perhead(cache, raw[:, :T].contiguous().cuda(), gate[:, :T].contiguous().cuda())
    for t in range(T, T + steps):
        csld.kv_cache_append_perhead(cache, raw[:, t].contiguous().cuda(), gate[:, t].contiguous().cuda())
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    bits = raw.view(torch.int16).numpy().view(np.uint16)
    g = gate.numpy()
    st = orc.LayerState(B, cache.capacity, m, W, True, key_heads=4)
    for t in range(T + steps):
        orc.append_batch(st, bias.numpy(), w, bits[:, t].copy(), g[:, t].copy())
    assert np.array_equal(cache.seq_len.cpu().numpy(), st.seq_len)
    n = (T + steps) // m
    H.assert_entries_close(cache.comp_kv[:, :n].cpu().numpy(), st.comp_kv[:, :n], "per-head cache entries",
                           H.pool_slack(raw, m))
    for b_ in range(B):
        _keys_close(_unswizzle(cache.ikeys[b_, :n].cpu().numpy()), cache.iscales[b_, :n].cpu().numpy(),
                    st.ikeys[b_, :n], st.iscales[b_, :n], lambda: _ramax(orc, bits[b_], g[b_], bias.numpy(), m, w, n))


def _random_perhead_keys(B, cap, seed):
    g = synth.gen(seed)
    keys = np.zeros((B, cap, 4, 32), np.uint8)
    scales = np.zeros((B, cap, 4, 2), np.float32)
    for h in range(4):
        ik, isc = synth.random_ikeys(B, cap, g, heavy_frac=0.01)
        keys[:, :, h], scales[:, :, h] = ik.numpy(), isc.numpy()
    return keys, scales


@pytest.mark.parametrize("B,cap,k,Q", [(4, 20000, 512, 1), (2, 262144, 1024, 1), (3, 9000, 256, 2), (5, 700, 1024, 1)])
def test_indexer_topk_perhead_matches_oracle(csld, orc, B, cap, k, Q):
    keys, scales = _random_perhead_keys(B, cap, seed=2200 + cap + Q)
    rng = np.random.default_rng(2201 + cap)
    q = rng.standard_normal((B, Q, 4, 64)).astype(np.float32)
    hw = np.abs(rng.standard_normal((B, Q, 4))).astype(np.float32)
    n_tok = np.array([4 * cap - 4 * (b_ * 37 % 200) for b_ in range(B)], np.int32)
    got = csld.indexer_topk_perhead(torch.from_numpy(_swizzle(keys)).cuda(), torch.from_numpy(scales).cuda(),
                                    torch.from_numpy(n_tok).cuda(), 4, torch.from_numpy(q).cuda(),
                                    torch.from_numpy(hw).cuda(), k)
    torch.cuda.synchronize()
    got = got.cpu().numpy()
    for j in range(Q):
        # query j sees the first n - Q + 1 + j tokens
        seq_j = n_tok - Q + 1 + j
        ref = orc.indexer_topk_batch_perhead(keys, scales, seq_j, 4, q[:, j].copy(), hw[:, j].copy(), k)
        H.assert_topk_equal(got[:, j], ref)
        for b_ in range(B):
            n = min(int(seq_j[b_]) // 4, cap)
            _, s64 = orc.indexer_scores_perhead(keys[b_, :n], scales[b_, :n], q[b_, j], hw[b_, j])
            sel64 = set(orc.topk64(s64, k).tolist()) - {-1}
            assert H.near_tie_only(set(got[b_, j].tolist()) - {-1}, sel64, s64)


def test_identical_heads_select_as_the_shared_key(csld):
    """W_h = W for every head: the per-head path selects exactly what the shared-key path does."""
    B, T, k = 2, 4 * 6000, 512
    parts = [synth.prefill_inputs(T, seed=2300 + b_) for b_ in range(B)]
    raw = torch.stack([p["raw"] for p in parts]).cuda()
    gate = torch.stack([p["gate"] for p in parts]).cuda()
    w = parts[0]["w_idx"]
    base = csld.LayerCache(B, T // 4 + 2, 4, 128, parts[0]["bias4"], w)
    ph = csld.LayerCache(B, T // 4 + 2, 4, 128, parts[0]["bias4"], w[:, None, :].repeat(1, 4, 1).contiguous(),
                         perhead=True)
    csld.kv_cache_prefill(base, raw, gate)
    csld.kv_cache_prefill_perhead(ph, raw, gate)
    qs = synth.decode_queries(B, seed=2301, device="cuda")
    a = csld.indexer_topk(base.ikeys, base.iscales, base.seq_len, 4, qs["q_idx"], qs["head_w"], k)
    b = csld.indexer_topk_perhead(ph.ikeys, ph.iscales, ph.seq_len, 4, qs["q_idx"][:, None].contiguous(),
                                  qs["head_w"][:, None].contiguous(), k)
    torch.cuda.synchronize()
    assert torch.equal(a, b[:, 0])
