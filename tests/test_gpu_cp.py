"""GPU parity of the context-parallel split of one sequence's compressed cache over R ranks,
emulated on one GPU: each rank is a host thread holding its own LayerCache with the entries of
its range, and the all-gathers between the ranks are stacks of their tensors (on the one
stream, so every rank's producer kernels precede the gather).  The merged selection must equal
the single-GPU indexer's bit for bit, and the merged attention the float64 oracle's within the
stated tolerance."""
import math
import threading

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


class _Exchange:
    """all_gather for R threads: each deposits its tensor, every thread gets the rank-ordered stack."""

    def __init__(self, R):
        self.R, self.slots, self.bar = R, [None] * R, threading.Barrier(R)

    def for_rank(self, r):
        def gather(t):
            self.slots[r] = t
            self.bar.wait()
            out = torch.stack(list(self.slots))
            self.bar.wait()
            return out
        return gather


def _run_ranks(R, fn):
    errs = []

    def wrap(r):
        try:
            fn(r)
        except Exception as e:   # noqa: BLE001 -- re-raised below
            errs.append(e)
            raise

    th = [threading.Thread(target=wrap, args=(r,)) for r in range(R)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=300)
    if errs:
        raise errs[0]


def _split_layer(csld, full, ratio, parts, r, W, bias, w_idx):
    lo, cnt = parts[r]
    B = full.batch
    cap = max(2, cnt + (cnt & 1))
    lay = csld.LayerCache(B, cap, ratio, W, bias, w_idx)
    lay.comp_kv[:, :cnt] = full.comp_kv[:, lo:lo + cnt]
    if full.has_indexer:
        # key bytes move with their entries; the stored layout depends on the entry index, so the
        # range start is a multiple of 8 and the bytes copy unchanged
        lay.ikeys[:, :cnt] = full.ikeys[:, lo:lo + cnt]
        lay.iscales[:, :cnt] = full.iscales[:, lo:lo + cnt]
    lay.win_kv.copy_(full.win_kv)
    lay.seq_len.fill_(cnt * ratio)
    return lay


@pytest.mark.parametrize("R,n,B,k", [(2, 4 * 20000 + 3, 2, 512), (4, 4 * 9000, 3, 256), (3, 4 * 700 + 1, 1, 1024)])
def test_context_parallel_csa_matches_single_gpu(csld, orc, R, n, B, k):
    W = 128
    inp = synth.prefill_inputs(8, seed=R)
    n_c = n // 4
    full = csld.LayerCache(B, n_c + 64, 4, W, inp["bias4"], inp["w_idx"])
    g = synth.gen(R * 7 + B)
    full.comp_kv[:, :n_c] = synth.random_entries((B, n_c), g).cuda()
    full.win_kv[:] = synth.random_entries((B, W), g).cuda()
    ik, isc = synth.random_ikeys(B, full.capacity, g, heavy_frac=0.01, n_valid=n_c)
    full.ikeys.copy_(synth.ikeys_swap_halves(ik).cuda())
    full.iscales.copy_(isc.cuda())
    full.seq_len.fill_(n)
    qs = synth.decode_queries(B, seed=R + 100, device="cuda")
    sel_full = csld.indexer_topk(full.ikeys, full.iscales, full.seq_len, 4, qs["q_idx"], qs["head_w"], k)
    parts = csld.partition_entries(n_c, R)
    rank_lo = torch.tensor([lo for lo, _ in parts], dtype=torch.int64, device="cuda")
    layers = [_split_layer(csld, full, 4, parts, r, W, inp["bias4"], inp["w_idx"]) for r in range(R)]
    ex = _Exchange(R)
    results, merged = [None] * R, [None] * R

    def rank(r):
        cp = csld.ContextParallelLayer(layers[r], parts[r][0], parts[r][1], rank_lo, window_rank=(r == R - 1),
                                       seq_len_total=full.seq_len, all_gather=ex.for_rank(r))
        results[r] = cp.step(qs["q"], SCALE, k=k, q_idx=qs["q_idx"], head_w=qs["head_w"])
        # the merged selection, as global indices, for the bit-exact check
        c = layers[r]
        sel = csld.indexer_topk(c.ikeys, c.iscales, c.seq_len, 4, qs["q_idx"], qs["head_w"], k)
        sc = csld.indexer_rescore(c.ikeys, c.iscales, qs["q_idx"], qs["head_w"], sel)
        g_sc, g_idx = cp.all_gather(sc), cp.all_gather(sel)
        merged[r] = csld.topk_merge(g_sc, g_idx, rank_lo, 0, n_c)       # the whole range: global indices

    _run_ranks(R, rank)
    torch.cuda.synchronize()
    for r in range(R):
        assert np.array_equal(merged[r].cpu().numpy(), sel_full.cpu().numpy()), f"rank {r}: merged top-k differs"
        assert torch.equal(results[r][0], results[0][0])
    out, lse = results[0]
    ro, rl = orc.attention_batch(synth.bits16(qs["q"].cpu()), full.comp_kv.cpu().numpy(), 4, sel_full.cpu().numpy(),
                                 full.win_kv.cpu().numpy(), full.seq_len.cpu().numpy(), SCALE)
    H.assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, f"context-parallel CSA over {R} ranks")


@pytest.mark.parametrize("R,n,B", [(2, 128 * 3000 + 5, 2), (4, 128 * 257, 3)])
def test_context_parallel_hca_matches_oracle(csld, orc, R, n, B):
    W = 128
    inp = synth.prefill_inputs(8, seed=R)
    n_c = n // 128
    full = csld.LayerCache(B, n_c + 8, 128, W, inp["bias128"])
    g = synth.gen(R * 11 + B)
    full.comp_kv[:, :n_c] = synth.random_entries((B, n_c), g).cuda()
    full.win_kv[:] = synth.random_entries((B, W), g).cuda()
    full.seq_len.fill_(n)
    q = synth.decode_queries(B, seed=R + 200, device="cuda")["q"]
    parts = csld.partition_entries(n_c, R)
    rank_lo = torch.tensor([lo for lo, _ in parts], dtype=torch.int64, device="cuda")
    layers = [_split_layer(csld, full, 128, parts, r, W, inp["bias128"], None) for r in range(R)]
    ex = _Exchange(R)
    results = [None] * R

    def rank(r):
        cp = csld.ContextParallelLayer(layers[r], parts[r][0], parts[r][1], rank_lo, window_rank=(r == R - 1),
                                       seq_len_total=full.seq_len, all_gather=ex.for_rank(r))
        results[r] = cp.step(q, SCALE)

    _run_ranks(R, rank)
    torch.cuda.synchronize()
    out, lse = results[0]
    ro, rl = orc.attention_batch(synth.bits16(q.cpu()), full.comp_kv.cpu().numpy(), 128, None,
                                 full.win_kv.cpu().numpy(), full.seq_len.cpu().numpy(), SCALE)
    H.assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, f"context-parallel HCA over {R} ranks")


def test_rescore_matches_oracle_scores(csld, orc):
    """indexer_rescore reproduces the oracle's fp32 score of every selected entry bit for bit."""
    B, n_c, k = 2, 5000, 300
    g = synth.gen(5)
    ik, isc = synth.random_ikeys(B, n_c, g)
    qs = synth.decode_queries(B, seed=6)
    sel = torch.stack([torch.randperm(n_c, generator=g)[:k] for _ in range(B)]).to(torch.int32)
    sel[0, :7] = -1
    got = csld.indexer_rescore(synth.ikeys_swap_halves(ik).cuda(), isc.cuda(), qs["q_idx"].cuda(),
                               qs["head_w"].cuda(), sel.cuda()).cpu().numpy()
    for b in range(B):
        s32, _ = orc.indexer_scores(ik[b].numpy(), isc[b].numpy(), qs["q_idx"][b].numpy(), qs["head_w"][b].numpy())
        s = sel[b].numpy()
        want = np.where(s >= 0, s32[np.maximum(s, 0)], -np.inf).astype(np.float32)
        assert np.array_equal(got[b], want)


def test_topk_merge_ties_and_padding(csld):
    """Equal scores go to the lower global index across ranks; fewer candidates than k pad -1."""
    R, B, k = 3, 1, 4
    sc = torch.tensor([[[5.0, 1.0, -np.inf, 2.0]], [[5.0, 3.0, 3.0, 0.0]], [[5.0, -1.0, 2.0, 2.0]]]).cuda()
    idx = torch.tensor([[[0, 1, -1, 3]], [[0, 1, 2, 3]], [[0, 1, 2, 3]]], dtype=torch.int32).cuda()
    lo = torch.tensor([0, 10, 20], dtype=torch.int64).cuda()
    got = csld.topk_merge(sc, idx, lo, 0, 100).cpu().numpy()
    assert got.tolist() == [[0, 10, 11, 20]]   # the three 5s, then 3 at index 11 before 3 at 12
