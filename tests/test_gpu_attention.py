"""GPU parity of hybrid_decode_attention (dense HCA mode and sparse CSA mode, each with the
sliding-window branch) against the float64 oracle: |gpu - oracle| <= 2e-2 + 1e-2 |oracle|."""
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


def _caches(B, cap, W, seed):
    g = synth.gen(seed)
    comp = synth.random_entries((B, cap), g)
    win = synth.random_entries((B, max(W, 1)), g)
    return comp, win


def _run(csld, orc, q, comp, ratio, sel, win, W, seq, scale=SCALE):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = csld.hybrid_decode_attention(q.cuda(), comp.cuda(), ratio,
                                            None if sel is None else sel.cuda(), win.cuda(), W,
                                            seq.cuda(), scale, err=err)
    torch.cuda.synchronize()
    ro, rl = orc.attention_batch(synth.bits16(q), comp.numpy(), ratio,
                                 None if sel is None else sel.numpy(), win.numpy()[:, :W] if W > 0 else
                                 np.zeros((q.shape[0], 0, 576), np.uint8), seq.numpy(), scale)
    return out.cpu().numpy(), lse.cpu().numpy(), ro, rl, err.item()


@pytest.mark.parametrize("B,n,W,ratio", [(1, 4096, 128, 128), (2, 128 * 64 + 5, 128, 128), (3, 1000, 64, 4),
                                         (1, 70, 128, 128), (2, 0, 16, 4), (1, 9, 0, 4), (2, 640, 1, 128),
                                         (1, 50000, 128, 4), (32, 128 * 600 + 7, 128, 128), (20, 4 * 3000, 64, 4),
                                         (100, 128 * 20 + 3, 32, 128), (200, 640, 16, 4)])
def test_dense_matches_oracle(csld, orc, B, n, W, ratio):
    cap = max(2, n // ratio + 8)
    comp, win = _caches(B, cap, W, seed=n + B)
    q = synth.decode_queries(B, seed=n)["q"]
    seq = torch.tensor([n - (b * 3 if n > 10 else 0) for b in range(B)], dtype=torch.int32)
    out, lse, ro, rl, err = _run(csld, orc, q, comp, ratio, None, win, W, seq)
    assert err == 0
    H.assert_attention_close(out, lse, ro, rl)
    if n == 0:
        assert np.all(out == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("B,n_c,k,W", [(1, 1024, 128, 128), (4, 32768, 512, 128), (2, 300, 512, 64), (3, 5000, 1, 8),
                                       (40, 5000, 1024, 128)])
def test_sparse_matches_oracle(csld, orc, B, n_c, k, W):
    cap = n_c + 16
    comp, win = _caches(B, cap, W, seed=k + n_c)
    q = synth.decode_queries(B, seed=k)["q"]
    g = synth.gen(3)
    sel = torch.full((B, k), -1, dtype=torch.int32)
    for b in range(B):
        m = min(k, n_c)
        sel[b, :m] = torch.sort(torch.randperm(n_c, generator=g)[:m]).values.to(torch.int32)
    seq = torch.full((B,), 4 * n_c + 2, dtype=torch.int32)
    out, lse, ro, rl, err = _run(csld, orc, q, comp, 4, sel, win, W, seq)
    assert err == 0
    H.assert_attention_close(out, lse, ro, rl)


def test_sparse_unordered_padded_and_bad_index(csld, orc):
    B, n_c, k, W = 2, 500, 64, 16
    comp, win = _caches(B, n_c + 4, W, seed=17)
    q = synth.decode_queries(B, seed=18)["q"]
    sel = torch.randint(0, n_c, (B, k), generator=synth.gen(19), dtype=torch.int32)
    sel[0, 10:20] = -1                                   # holes anywhere
    sel[1, 5] = n_c + 1                                  # not a visible entry: flagged and skipped
    seq = torch.full((B,), 4 * n_c, dtype=torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = csld.hybrid_decode_attention(q.cuda(), comp.cuda(), 4, sel.cuda(), win.cuda(), W,
                                            seq.cuda(), SCALE, err=err)
    torch.cuda.synchronize()
    assert err.item() & 2
    ref_sel = sel.clone()
    ref_sel[1, 5] = -1
    ro, rl = orc.attention_batch(synth.bits16(q), comp.numpy(), 4, ref_sel.numpy(), win.numpy(),
                                 seq.numpy(), SCALE)
    H.assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), ro, rl)


@pytest.mark.parametrize("scale", [0.01, 0.3, 1.0])
def test_scale_and_large_logits(csld, orc, scale):
    B, n, W = 2, 128 * 40, 128
    comp, win = _caches(B, n // 128 + 2, W, seed=23)
    q = (synth.decode_queries(B, seed=24)["q"].float() * 3).to(torch.bfloat16)
    seq = torch.full((B,), n, dtype=torch.int32)
    out, lse, ro, rl, err = _run(csld, orc, q, comp, 128, None, win, W, seq, scale)
    H.assert_attention_close(out, lse, ro, rl)


@pytest.mark.parametrize("name", ["decode128k", "decode1m"])
def test_full_workload_dense_and_sparse(csld, orc, name):
    wl = synth.WORKLOADS[name]
    B = wl.batch
    g = synth.gen(29)
    hca = synth.random_entries((B, wl.hca_cap), g)
    win = synth.random_entries((B, wl.window), g)
    q = synth.decode_queries(B, seed=30)["q"]
    seq = torch.full((B,), wl.context, dtype=torch.int32)
    out, lse, ro, rl, err = _run(csld, orc, q, hca, wl.hca_ratio, None, win, wl.window, seq)
    assert err == 0
    H.assert_attention_close(out, lse, ro, rl, f"{name} HCA")
    # CSA: a sample of 2 sequences' caches at full size, top-k of random valid indices
    Bs = 2
    csa = synth.random_entries((Bs, wl.csa_cap), g)
    sel = torch.stack([torch.sort(torch.randperm(wl.csa_entries, generator=g)[:wl.topk]).values
                       for _ in range(Bs)]).to(torch.int32)
    out, lse, ro, rl, err = _run(csld, orc, q[:Bs].contiguous(), csa, wl.csa_ratio, sel, win[:Bs].contiguous(),
                                 wl.window, seq[:Bs].contiguous())
    assert err == 0
    H.assert_attention_close(out, lse, ro, rl, f"{name} CSA")



@pytest.mark.parametrize("mode", ["hca", "csa"])
def test_full_workload_peaked_softmax(csld, orc, mode):
    """The 1M-token workload (B = 8) with a peaked softmax: a few hundred entries per sequence
    aligned with the query, so a weight or value error of a few percent fails the bar."""
    wl = synth.WORKLOADS["decode1m"]
    B = wl.batch
    g = synth.gen(31)
    q = synth.decode_queries(B, seed=32)["q"]
    win = synth.random_entries((B, wl.window), g)
    seq = torch.full((B,), wl.context, dtype=torch.int32)
    if mode == "hca":
        comp = synth.random_entries((B, wl.hca_cap), g)
        idx = [torch.randperm(wl.hca_entries, generator=g)[:256] for _ in range(B)]
        sel, ratio = None, wl.hca_ratio
    else:
        B = 2
        q, win, seq = q[:B].contiguous(), win[:B].contiguous(), seq[:B].contiguous()
        comp = synth.random_entries((B, wl.csa_cap), g)
        sel = torch.stack([torch.sort(torch.randperm(wl.csa_entries, generator=g)[:wl.topk]).values
                           for _ in range(B)]).to(torch.int32)
        idx = [sel[b, torch.randperm(wl.topk, generator=g)[:256]].long() for b in range(B)]
        ratio = wl.csa_ratio
    H.plant_aligned(comp, q, idx, g)
    out, lse, ro, rl, err = _run(csld, orc, q, comp, ratio, sel, win, wl.window, seq)
    assert err == 0
    assert np.abs(ro).max() > 0.5 and np.median(np.abs(ro)) > 0.05   # the case really is peaked
    H.assert_attention_close(out, lse, ro, rl, f"decode1m {mode} peaked")
