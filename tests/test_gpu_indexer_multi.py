"""GPU parity of the multi-query lightning indexer (several query tokens of a sequence scored in
one pass over the FP4 keys): query j of sequence b, at raw position seq_len - Q + j, must get
exactly the oracle's fp32 selection over the entries it can see, and the stated float64 rule
(ties to the lower index, near-ties < 1e-6 exempt), and the same set the single-query
indexer_topk gives it."""
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


def _queries(B, Q, seed):
    g = synth.gen(seed)
    q = torch.randn((B, Q, 4, 64), generator=g)
    w = torch.randn((B, Q, 4), generator=g).abs()
    return q, w


@pytest.mark.parametrize("B,Q,n,k,ratio", [(2, 8, 4 * 20000 + 3, 512, 4), (3, 5, 4 * 3000, 256, 4),
                                           (1, 1, 4 * 1500 + 2, 128, 4), (4, 8, 4 * 600, 1024, 4),
                                           (2, 3, 9 * 2000 + 4, 100, 9), (1, 8, 4 * 262144, 1024, 4),
                                           (8, 4, 4 * 262144, 1024, 4)])
def test_multi_query_matches_oracle_and_single_query(csld, orc, B, Q, n, k, ratio):
    n_c = n // ratio
    cap = n_c + 64
    g = synth.gen(n + Q)
    ik, isc = synth.random_ikeys(B, cap, g, heavy_frac=0.01, n_valid=n_c)
    q, w = _queries(B, Q, seed=Q * 13 + B)
    seq = torch.full((B,), n, dtype=torch.int32)
    seq[-1] = n - 7 if B > 1 else n               # a ragged batch
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dk = synth.ikeys_swap_halves(ik).cuda()
    out = csld.indexer_topk_multi(dk, isc.cuda(), seq.cuda(), ratio, q.cuda(), w.cuda(), k, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    for j in range(Q):
        pos1 = (seq - Q + j + 1).to(torch.int32)  # tokens query j sees
        ref = orc.indexer_topk_batch(ik.numpy(), isc.numpy(), pos1.numpy(), ratio, q[:, j].contiguous().numpy(),
                                     w[:, j].contiguous().numpy(), k)
        H.assert_topk_equal(got[:, j], ref)
        H.assert_topk_matches_f64(orc, got[:, j], ik.numpy(), isc.numpy(), pos1.numpy(), ratio,
                                  q[:, j].contiguous().numpy(), w[:, j].contiguous().numpy(), k)
        single = csld.indexer_topk(dk, isc.cuda(), pos1.cuda(), ratio, q[:, j].contiguous().cuda(),
                                   w[:, j].contiguous().cuda(), k)
        assert np.array_equal(single.cpu().numpy(), got[:, j])


def test_multi_query_ties_short_sequences_and_reuse(csld, orc):
    """Identical keys (ties to the lower index), sequences shorter than Q tokens or than k
    entries, and one workspace reused across calls."""
    B, Q, k, cap = 3, 4, 64, 4000
    ik = torch.full((B, cap, 32), 0x22, dtype=torch.uint8)
    ik[0, 1000:1030] = 0x44
    isc = torch.ones((B, cap, 2), dtype=torch.float32)
    q = torch.ones((B, Q, 4, 64))
    w = torch.ones((B, Q, 4))
    ws = csld.indexer_multi_workspace(B, Q, cap)
    for seq_vals in ([4 * cap, 4 * 50 + 2, 2], [4 * 3000, 4 * 64 + 3, 4 * cap]):
        seq = torch.tensor(seq_vals, dtype=torch.int32)
        got = csld.indexer_topk_multi(synth.ikeys_swap_halves(ik).cuda(), isc.cuda(), seq.cuda(), 4, q.cuda(),
                                      w.cuda(), k, ws=ws).cpu().numpy()
        for j in range(Q):
            pos1 = (seq - Q + j + 1).clamp_min(0).to(torch.int32)
            ref = orc.indexer_topk_batch(ik.numpy(), isc.numpy(), pos1.numpy(), 4, q[:, j].contiguous().numpy(),
                                         w[:, j].contiguous().numpy(), k)
            H.assert_topk_equal(got[:, j], ref)
