"""GPU parity of multi-query decode attention (Q draft tokens per sequence, as in multi-token
prediction or speculative decoding): query j of sequence b sees the first seq_len - Q + 1 + j
tokens -- the compressed entries they complete (dense mode) or its own top-k row (sparse mode),
and the W newest of them through a window ring of W_ring >= W + Q - 1 slots.  Each query is
checked against the float64 oracle run for that query alone."""
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


def _ring_for(ring, n_j, W, W_ring):
    """The window ring the oracle expects for a query that sees n_j tokens: W slots, token t at
    slot t mod W, holding tokens max(0, n_j - W) .. n_j - 1 taken from the big ring."""
    out = np.zeros((W, 576), np.uint8)
    for t in range(max(0, n_j - W), n_j):
        out[t % W] = ring[t % W_ring]
    return out


@pytest.mark.parametrize("mode,B,Q,n,W,ratio,k", [("dense", 2, 4, 128 * 300 + 2, 128, 128, 0),
                                                  ("dense", 3, 8, 128 * 2 + 5, 128, 128, 0),
                                                  ("sparse", 2, 4, 4 * 5000 + 1, 128, 4, 512),
                                                  ("sparse", 1, 3, 4 * 800, 64, 4, 128),
                                                  ("dense", 2, 2, 70, 128, 128, 0)])
def test_multi_query_attention_matches_oracle(csld, orc, mode, B, Q, n, W, ratio, k):
    W_ring = W + Q - 1
    n_c = n // ratio
    cap = n_c + 8
    g = synth.gen(n + Q + B)
    comp = synth.random_entries((B, cap), g)
    ring = synth.random_entries((B, W_ring), g)
    q = synth.decode_queries(B * Q, seed=Q + n)["q"].view(B, Q, 16, 512).contiguous()
    seq = torch.full((B,), n, dtype=torch.int32)
    sel = None
    if mode == "sparse":
        sel = torch.full((B, Q, k), -1, dtype=torch.int32)
        for b in range(B):
            for j in range(Q):
                vis = (n - (Q - 1 - j)) // ratio
                m = min(k, vis)
                sel[b, j, :m] = torch.sort(torch.randperm(vis, generator=g)[:m]).values.to(torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = csld.hybrid_decode_attention_multi(q.cuda(), comp.cuda(), ratio, None if sel is None else sel.cuda(),
                                                  ring.cuda(), W, seq.cuda(), SCALE, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for j in range(Q):
        n_j = n - (Q - 1 - j)
        rings = np.stack([_ring_for(ring[b].numpy(), n_j, W, W_ring) for b in range(B)])
        ro, rl = orc.attention_batch(synth.bits16(q[:, j].contiguous()), comp.numpy(), ratio,
                                     None if sel is None else sel[:, j].contiguous().numpy(), rings,
                                     np.full(B, n_j, np.int32), SCALE)
        H.assert_attention_close(out[:, j], lse[:, j], ro, rl, f"{mode} query {j} of {Q}")


def test_multi_query_window_only_block(csld, orc):
    """The multi-token-prediction block attends the window only: no compressed entry is visible
    to any of the Q queries (fewer tokens than one block)."""
    B, Q, W = 2, 4, 128
    n = 100
    W_ring = W + Q - 1
    g = synth.gen(3)
    comp = synth.random_entries((B, 2), g)
    ring = synth.random_entries((B, W_ring), g)
    q = synth.decode_queries(B * Q, seed=4)["q"].view(B, Q, 16, 512).contiguous()
    seq = torch.full((B,), n, dtype=torch.int32)
    out, lse = csld.hybrid_decode_attention_multi(q.cuda(), comp.cuda(), 128, None, ring.cuda(), W, seq.cuda(), SCALE)
    torch.cuda.synchronize()
    for j in range(Q):
        n_j = n - (Q - 1 - j)
        rings = np.stack([_ring_for(ring[b].numpy(), n_j, W, W_ring) for b in range(B)])
        ro, rl = orc.attention_batch(synth.bits16(q[:, j].contiguous()), comp.numpy(), 128, None, rings,
                                     np.full(B, n_j, np.int32), SCALE)
        H.assert_attention_close(out[:, j].cpu().numpy(), lse[:, j].cpu().numpy(), ro, rl, f"window-only query {j}")


@pytest.mark.parametrize("mode", ["dense", "sparse"])
def test_multi_query_full_size_peaked(csld, orc, mode):
    """The multi-token workload at full size: 4 query tokens per sequence at 1M tokens, dense over
    the 8,192 HCA entries of all 8 sequences (the last query alone sees entry 8,191), or sparse
    over each query's own top-1024 of 262,144 CSA entries (2 sequences); window 128 in a ring of
    131 slots.  128 entries per query are aligned with that query's heads, so every softmax is
    peaked and a weight or value error of a few percent fails the bar."""
    wl = synth.WORKLOADS["decode1m"]
    Q, W, n = 4, wl.window, wl.context
    W_ring = W + Q - 1
    g = synth.gen(77)
    B = wl.batch if mode == "dense" else 2
    ratio = wl.hca_ratio if mode == "dense" else wl.csa_ratio
    comp = synth.random_entries((B, wl.hca_cap if mode == "dense" else wl.csa_cap), g)
    ring = synth.random_entries((B, W_ring), g)
    q = synth.decode_queries(B * Q, seed=78)["q"].view(B, Q, 16, 512).contiguous()
    seq = torch.full((B,), n, dtype=torch.int32)
    sel = None
    if mode == "sparse":
        sel = torch.stack([torch.stack([torch.sort(torch.randperm((n - (Q - 1 - j)) // ratio, generator=g)[:wl.topk]).values
                                        for j in range(Q)]) for _ in range(B)]).to(torch.int32)
    for j in range(Q):
        if mode == "sparse":
            idx = [sel[b, j, torch.randperm(wl.topk, generator=g)[:128]].long() for b in range(B)]
        else:
            idx = [torch.randperm(wl.hca_entries, generator=g)[:128] for _ in range(B)]
        H.plant_aligned(comp, q[:, j], idx, g)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = csld.hybrid_decode_attention_multi(q.cuda(), comp.cuda(), ratio, None if sel is None else sel.cuda(),
                                                  ring.cuda(), W, seq.cuda(), SCALE, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for j in range(Q):
        n_j = n - (Q - 1 - j)
        rings = np.stack([_ring_for(ring[b].numpy(), n_j, W, W_ring) for b in range(B)])
        ro, rl = orc.attention_batch(synth.bits16(q[:, j].contiguous()), comp.numpy(), ratio,
                                     None if sel is None else sel[:, j].contiguous().numpy(), rings,
                                     np.full(B, n_j, np.int32), SCALE)
        assert np.abs(ro).max() > 0.5 and np.median(np.abs(ro)) > 0.05   # the case really is peaked
        H.assert_attention_close(out[:, j], lse[:, j], ro, rl, f"mtp1m {mode} query {j} of {Q}")
