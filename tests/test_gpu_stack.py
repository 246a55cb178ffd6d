"""GPU parity of the 61-layer hybrid stack (layers 0-1 HCA, then CSA / HCA alternating from
layer 2; "DeepSeek-V4: a million-token context that agents can actually use", layer-pattern
paragraph): every layer gets its own prefilled cache, one decode step runs through all of them
(append, indexer top-k and sparse attention on CSA layers, dense attention on HCA layers), and
a seeded sample of (layer, sequence) slices is checked against the float64 oracle run on the
same cache bytes."""
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


def test_layer_pattern(csld):
    kinds = csld.layer_pattern(61)
    assert kinds[:2] == ["hca", "hca"] and kinds[2] == "csa" and kinds.count("csa") == 30
    assert all(kinds[i] != kinds[i + 1] for i in range(2, 60))


@pytest.mark.parametrize("ctx,B,k", [(65536 - 3, 2, 512), (4096 + 77, 3, 128), (1 << 20, 8, 1024)])
def test_stack_step_matches_oracle_on_sampled_layers(csld, orc, ctx, B, k):
    """One decode step through all 61 layers (each prefilled from its own raw tokens), checked on
    sampled (layer, sequence) slices.  The 1M-token, batch-8 case is the sweep's headline point in
    the bench's launch configuration (about 40 GB of caches)."""
    # caches (CSA entries and keys on half the layers), the raw tokens of one layer, and the fp32
    # draws of one sequence, roughly
    need = 61 * B * (ctx // 4) * 616 // 2 + 2 * B * ctx * 512 + 8 * ctx * 512 + (1 << 30)
    if torch.cuda.mem_get_info()[0] < need:
        pytest.skip(f"needs about {need / 1e9:.0f} GB of free device memory")
    kinds = csld.layer_pattern(61)
    L, W = len(kinds), 128
    inp = synth.prefill_inputs(8, seed=1)
    st = csld.DecodeStack(B, kinds, (ctx + 64) // 4, (ctx + 256) // 128, W, k, inp["bias4"], inp["bias128"],
                          inp["w_idx"])
    g = synth.gen(2, "cuda")
    raw = torch.empty((B, ctx, 512), dtype=torch.bfloat16, device="cuda")
    for lay in st.layers:   # a distinct prefill per layer
        for b in range(B):
            raw[b] = synth.bf16_normal((ctx, 512), g, "cuda")
        gate = torch.randn((B, ctx), generator=g, device="cuda")
        csld.kv_cache_prefill(lay, raw, gate)
    del raw, gate
    toks = synth.decode_tokens(L * B, seed=3, device="cuda")
    qs = synth.decode_queries(L * B, seed=4, device="cuda")
    kv_new, gate_new = toks["kv"].view(L, B, 512), toks["gate"].view(L, B)
    q, q_idx, head_w = qs["q"].view(L, B, 16, 512), qs["q_idx"].view(L, B, 4, 64), qs["head_w"].view(L, B, 4)
    out = torch.empty((L, B, 16, 512), dtype=torch.float32, device="cuda")
    lse = torch.empty((L, B, 16), dtype=torch.float32, device="cuda")
    st.step(kv_new, gate_new, q, q_idx, head_w, SCALE, out, lse)
    torch.cuda.synchronize()
    assert st.err.item() == 0
    rng = np.random.default_rng(ctx)
    sample = sorted(set([0, 1, 2, 3, L - 2, L - 1] + list(rng.choice(L, 4, replace=False))))
    for i in sample:
        lay = st.layers[i]
        assert int(lay.seq_len[0].item()) == ctx + 1
        b = int(rng.integers(B))
        sl = slice(b, b + 1)
        qb = synth.bits16(q[i, sl].cpu())
        comp = lay.comp_kv[sl].cpu().numpy()
        win = lay.win_kv[sl].cpu().numpy()
        seq = lay.seq_len[sl].cpu().numpy()
        if lay.has_indexer:
            keys = synth.ikeys_swap_halves(lay.ikeys[sl].cpu().numpy())
            osel = orc.indexer_topk_batch(keys, lay.iscales[sl].cpu().numpy(), seq, 4, q_idx[i, sl].cpu().numpy(),
                                          head_w[i, sl].cpu().numpy(), k)
            H.assert_topk_matches_f64(orc, osel, keys, lay.iscales[sl].cpu().numpy(), seq, 4,
                                      q_idx[i, sl].cpu().numpy(), head_w[i, sl].cpu().numpy(), k)
            ro, rl = orc.attention_batch(qb, comp, 4, osel, win, seq, SCALE)
        else:
            ro, rl = orc.attention_batch(qb, comp, 128, None, win, seq, SCALE)
        H.assert_attention_close(out[i, sl].cpu().numpy(), lse[i, sl].cpu().numpy(), ro, rl,
                                 f"layer {i} ({kinds[i]}) sequence {b}")


def test_stack_kv_bytes_against_gqa8(csld):
    """The stack's cache at 1M tokens is about 2 % of a GQA-8 bf16 cache (head dim 128)."""
    kinds = csld.layer_pattern(61)
    inp = synth.prefill_inputs(8, seed=1)
    st = csld.DecodeStack(1, kinds, 64, 8, 128, 16, inp["bias4"], inp["bias128"], inp["w_idx"])
    n = 1 << 20
    frac = st.kv_bytes_per_sequence(n) / (61 * n * 4096)
    assert 0.0190 < frac < 0.0191, frac
