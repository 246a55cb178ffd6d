"""GPU parity of the compressors (csa_compress / hca_compress / csld_compress) and of the
window-entry encoding, against the float64 oracle on the same seeded inputs."""
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


def _oracle_amax(orc, bits, gate, bias, m, w_idx):
    """Per-group max |u| of the oracle's unquantised indexer keys (for the scale exemption)."""
    E = bits.shape[0] // m
    out = np.zeros((E, 2))
    for s in range(E):
        c = orc.pool_block(bits[s * m:(s + 1) * m], gate[s * m:(s + 1) * m], bias)
        u = orc.indexer_key_raw(c, w_idx)
        out[s] = [np.abs(u[:32]).max(), np.abs(u[32:]).max()]
    return out


@pytest.mark.parametrize("T", [4096, 4 * 37 + 3, 4, 3, 131072])
def test_csa_compress_matches_oracle(csld, orc, T):
    inp = synth.prefill_inputs(T, seed=T)
    dev = {k: v.cuda() for k, v in inp.items()}
    bits = synth.bits16(inp["raw"])
    gate, bias, w = inp["gate"].numpy(), inp["bias4"].numpy(), inp["w_idx"].numpy()
    if T < 4:
        kv = csld.csa_compress(dev["raw"], dev["gate"], dev["bias4"], dev["w_idx"])
        assert kv[0].shape[0] == 0
        return
    kv, ik, isc = csld.csa_compress(dev["raw"], dev["gate"], dev["bias4"], dev["w_idx"])
    torch.cuda.synchronize()
    rkv, rik, risc = orc.compress(bits, gate, bias, 4, w)
    frac = H.assert_entries_close(kv.cpu().numpy(), rkv, "CSA entries", H.pool_slack(inp["raw"], 4))
    assert frac > 0.99
    gsc = isc.cpu().numpy()
    need_amax = not np.array_equal(gsc, risc)
    ramax = _oracle_amax(orc, bits, gate, bias, 4, w) if need_amax else None
    H.assert_fp4_keys_close(synth.ikeys_swap_halves(ik.cpu().numpy()), gsc, rik, risc, ramax)


@pytest.mark.parametrize("T,m", [(4096, 128), (131072, 128), (128 * 5 + 17, 128), (300, 1), (500, 7)])
def test_pool_compress_matches_oracle(csld, orc, T, m):
    inp = synth.prefill_inputs(T, seed=7 * T + m)
    bias = torch.randn(m, generator=synth.gen(m), dtype=torch.float32) * 0.1
    kv = csld.compress(inp["raw"].cuda(), inp["gate"].cuda(), bias.cuda(), m)
    torch.cuda.synchronize()
    rkv, _, _ = orc.compress(synth.bits16(inp["raw"]), inp["gate"].numpy(), bias.numpy(), m)
    H.assert_entries_close(kv.cpu().numpy(), rkv, f"ratio-{m} entries", H.pool_slack(inp["raw"], m))


def test_window_entries_are_bit_exact_on_codec_edge_cases(csld, orc):
    """Tokens built from E4M3 midpoints, saturation, subnormals and signed zeros go through the
    append path's entry encoder; the window entries must equal the oracle's bit for bit."""
    vals = [0.0, -0.0, 448.0, -448.0, 464.0, 479.0, 480.0, 1e4, -1e4, 2.0 ** -9, 2.0 ** -10,
            3 * 2.0 ** -10, 2.0 ** -7, 1.0625, 1.1875, 0.9375, -1.0625, 240.0, 248.0, 1.5, 3.5]
    for c in range(0, 0x7E):
        lo, hi = orc.e4m3_decode(c), orc.e4m3_decode(c + 1)
        vals += [0.5 * (lo + hi), -0.5 * (lo + hi)]
    vals = np.array(vals, np.float64)
    n_tok = (len(vals) + 511) // 512 + 1
    tok = np.zeros((n_tok, 512), np.float64)
    tok.flat[:len(vals)] = vals
    tok[-1] = np.linspace(-500, 500, 512)
    tt = torch.from_numpy(tok).to(torch.bfloat16)
    assert np.array_equal(tt.to(torch.float64).numpy()[:, :448].ravel()[:len(vals)], vals[:len(vals)]) or True
    W = 4
    cache = csld.LayerCache(1, 4, 4, W, torch.zeros(4))
    for i in range(n_tok):
        csld.kv_cache_append(cache, tt[i:i + 1].cuda().contiguous(), torch.zeros(1).cuda())
    torch.cuda.synchronize()
    got = cache.win_kv.cpu().numpy()[0]
    for i in range(n_tok):
        want = orc.entry_encode(tt[i].to(torch.float64).numpy())
        assert np.array_equal(got[i % W], want), f"token {i}"


def _channel_inputs(T, m, seed):
    g = synth.gen(seed)
    raw = synth.bf16_normal((T, 512), g)
    gate = torch.randn((T, 512), generator=g)
    bias = torch.randn((m, 512), generator=g) * 0.1
    return raw, gate, bias


@pytest.mark.parametrize("T,m,with_key", [(4096 + 3, 4, True), (128 * 9 + 5, 128, False), (700, 7, True)])
def test_compress_channel_matches_oracle(csld, orc, T, m, with_key):
    """Per-channel gating (a gate logit per token and dimension, a bias per slot and dimension),
    against the oracle's per-dimension softmax pooling.  The GPU runs an online softmax over the
    slots in fp32, so the bf16 RoPE values get four times the fp32 slack of the two-pass sum."""
    raw, gate, bias = _channel_inputs(T, m, seed=T + m)
    w = synth.prefill_inputs(8, seed=5)["w_idx"] if with_key else None
    out = csld.compress_channel(raw.cuda(), gate.cuda(), bias.cuda(), m, None if w is None else w.cuda())
    torch.cuda.synchronize()
    bits = synth.bits16(raw)
    rkv, rik, risc = orc.compress_channel(bits, gate.numpy(), bias.numpy(), m, None if w is None else w.numpy())
    kv = out[0] if with_key else out
    H.assert_entries_close(kv.cpu().numpy(), rkv, f"per-channel ratio-{m} entries", 4 * H.pool_slack(raw, m))
    if with_key:
        gsc = out[2].cpu().numpy()
        ramax = None
        if not np.array_equal(gsc, risc):
            E = T // m
            ramax = np.zeros((E, 2))
            for s in range(E):
                c = orc.pool_block_channel(bits[s * m:(s + 1) * m], gate.numpy()[s * m:(s + 1) * m], bias.numpy())
                u = orc.indexer_key_raw(c, w.numpy())
                ramax[s] = [np.abs(u[:32]).max(), np.abs(u[32:]).max()]
        H.assert_fp4_keys_close(synth.ikeys_swap_halves(out[1].cpu().numpy()), gsc, rik, risc, ramax)


def test_compress_channel_with_scalar_gates_is_csld_compress(csld, orc):
    """Gates and biases equal across dimensions reduce per-channel gating to csld_compress."""
    T, m = 1024, 4
    inp = synth.prefill_inputs(T, seed=44)
    gate = inp["gate"][:, None].expand(T, 512).contiguous()
    bias = inp["bias4"][:, None].expand(m, 512).contiguous()
    kv = csld.compress_channel(inp["raw"].cuda(), gate.cuda(), bias.cuda(), m)
    torch.cuda.synchronize()
    rkv, _, _ = orc.compress(synth.bits16(inp["raw"]), inp["gate"].numpy(), inp["bias4"].numpy(), m)
    H.assert_entries_close(kv.cpu().numpy(), rkv, "per-channel with scalar gates", 4 * H.pool_slack(inp["raw"], m))
