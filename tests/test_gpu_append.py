"""GPU parity of kv_cache_prefill / kv_cache_append (window ring, tail, compressed entries and
indexer keys, lengths) against the oracle's token-by-token append, plus capacity handling."""
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


def _oracle_state(orc, bits, gates, m, W, cap, bias, w_idx):
    B, T = bits.shape[0], bits.shape[1]
    st = orc.LayerState(B, cap, m, W, w_idx is not None)
    for t in range(T):
        orc.append_batch(st, bias, w_idx, bits[:, t].copy(), gates[:, t].copy())
    return st


def _ramax(orc, bits, gates, bias, m, w_idx, b, n):
    out = np.zeros((n, 2))
    for s in range(n):
        c = orc.pool_block(bits[b, s * m:(s + 1) * m], gates[b, s * m:(s + 1) * m], bias)
        u = orc.indexer_key_raw(c, w_idx)
        out[s] = [np.abs(u[:32]).max(), np.abs(u[32:]).max()]
    return out


def _compare_ring_and_tail(cache, win_ref, tail_ref, gate_ref, seq_len):
    """Only the live slots are state: ring slots of the last min(W, n) tokens and the tail
    slots of the block being filled (t mod m < n mod m); the others are don't-care."""
    W, m = cache.window, cache.ratio
    win = cache.win_kv.cpu().numpy()
    tail = cache.tail_kv.view(torch.int16).cpu().numpy().view(np.uint16)
    tg = cache.tail_gate.cpu().numpy()
    for b, n in enumerate(np.asarray(seq_len).tolist()):
        for t in range(max(0, n - W), n):
            assert np.array_equal(win[b, t % W], win_ref[b, t % W]), f"window slot of token {t}"
        for j in range(n % m):
            assert np.array_equal(tail[b, j], tail_ref[b, j]) and tg[b, j] == gate_ref[b, j], f"tail slot {j}"


def _compare(cache, st, with_idx, ramax_fn=None, slack=0.0):
    assert np.array_equal(cache.seq_len.cpu().numpy(), st.seq_len)
    H.assert_entries_close(cache.comp_kv.cpu().numpy(), st.comp_kv, "compressed entries", slack)
    _compare_ring_and_tail(cache, st.win_kv, st.tail_kv, st.tail_gate, st.seq_len)
    if with_idx:
        n = st.seq_len.min() // cache.ratio
        for b in range(cache.batch):
            gs = cache.iscales[b, :n].cpu().numpy()
            ramax = ramax_fn(b, n) if not np.array_equal(gs, st.iscales[b, :n]) else None
            H.assert_fp4_keys_close(synth.ikeys_swap_halves(cache.ikeys[b, :n].cpu().numpy()), gs, st.ikeys[b, :n],
                                    st.iscales[b, :n], ramax=ramax)


@pytest.mark.parametrize("m,W,idx,T,steps", [(4, 128, True, 4080, 16), (128, 128, False, 4080, 16),
                                             (4, 8, True, 13, 9), (128, 32, False, 100, 40),
                                             (1, 4, False, 5, 3)])
def test_prefill_then_append_matches_oracle(csld, orc, m, W, idx, T, steps):
    B = 2
    inp = synth.prefill_inputs(T + steps, seed=T + m)
    raw = torch.stack([inp["raw"], synth.prefill_inputs(T + steps, seed=T + m + 1)["raw"]])
    gate = torch.stack([inp["gate"], inp["gate"].flip(0).contiguous()])
    bias = inp["bias4"] if m == 4 else (inp["bias128"] if m == 128 else torch.zeros(m))
    w_idx = inp["w_idx"] if idx else None
    cap = (T + steps) // m + 2
    cache = csld.LayerCache(B, cap, m, W, bias, w_idx)
    csld.kv_cache_prefill(cache, raw[:, :T].contiguous().cuda(), gate[:, :T].contiguous().cuda())
    for t in range(T, T + steps):
        csld.kv_cache_append(cache, raw[:, t].contiguous().cuda(), gate[:, t].contiguous().cuda())
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    bits = raw.view(torch.int16).numpy().view(np.uint16)
    st = _oracle_state(orc, bits, gate.numpy(), m, W, cache.capacity, bias.numpy(),
                       None if w_idx is None else w_idx.numpy())
    _compare(cache, st, idx, lambda b_, n_: _ramax(orc, bits, gate.numpy(), bias.numpy(), m,
                                                   w_idx.numpy(), b_, n_), H.pool_slack(raw, m))


def test_append_equals_prefill_on_gpu(csld):
    """Appending token by token gives the same entry bytes as the prefill (same pooling code)."""
    T, m, W = 4 * 64 + 2, 4, 16
    inp = synth.prefill_inputs(T, seed=41)
    raw = inp["raw"][None].contiguous().cuda()
    gate = inp["gate"][None].contiguous().cuda()
    a = csld.LayerCache(1, T // m + 2, m, W, inp["bias4"], inp["w_idx"])
    b = csld.LayerCache(1, T // m + 2, m, W, inp["bias4"], inp["w_idx"])
    csld.kv_cache_prefill(a, raw, gate)
    for t in range(T):
        csld.kv_cache_append(b, raw[:, t].contiguous(), gate[:, t].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(a.comp_kv, b.comp_kv)
    assert torch.equal(a.seq_len, b.seq_len)
    _compare_ring_and_tail(a, b.win_kv.cpu().numpy(), b.tail_kv.view(torch.int16).cpu().numpy().view(np.uint16),
                           b.tail_gate.cpu().numpy(), b.seq_len.cpu().numpy())
    H.assert_fp4_keys_close(synth.ikeys_swap_halves(a.ikeys[0].cpu().numpy()), a.iscales[0].cpu().numpy(),
                            synth.ikeys_swap_halves(b.ikeys[0].cpu().numpy()), b.iscales[0].cpu().numpy(),
                            ramax=np.full((a.capacity, 2), 6.0))


def test_capacity_overflow_sets_flag_and_changes_nothing(csld):
    m, W = 4, 4
    inp = synth.prefill_inputs(12, seed=43)
    cache = csld.LayerCache(1, 1, m, W, inp["bias4"])       # room for entry 0 only
    for t in range(7):
        csld.kv_cache_append(cache, inp["raw"][t:t + 1].contiguous().cuda(), inp["gate"][t:t + 1].contiguous().cuda())
    torch.cuda.synchronize()
    snap = (cache.win_kv.clone(), cache.tail_kv.clone(), cache.seq_len.clone(), cache.comp_kv.clone())
    assert cache.err.item() == 0
    csld.kv_cache_append(cache, inp["raw"][7:8].contiguous().cuda(), inp["gate"][7:8].contiguous().cuda())
    torch.cuda.synchronize()
    assert cache.err.item() & 1
    assert torch.equal(snap[0], cache.win_kv) and torch.equal(snap[1], cache.tail_kv)
    assert torch.equal(snap[2], cache.seq_len) and torch.equal(snap[3], cache.comp_kv)
