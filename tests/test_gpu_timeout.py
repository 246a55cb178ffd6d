"""Recovery from a bounded wait that runs out, without any GPU fault: a test hook raises the
arrival targets of the cooperative indexer's cross-CTA barriers by one, so no barrier can be
met.  Each wait gives up after about half a second; the kernel must return, report
CSLD_DEVERR_TIMEOUT in the error word and leave the device usable, and after the workspace is
zero-filled again the same call must give the oracle's selection."""
import time

import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu
CSLD_DEVERR_TIMEOUT = 8


@pytest.fixture(scope="module")
def csld():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_long_decode_b200 as m
    return m


def test_indexer_barrier_timeout_then_recovery(csld, orc):
    B, cap, k = 2, 40000, 256          # the cooperative path: 2 x 53 ranges, all resident
    g = synth.gen(61)
    ik, isc = synth.random_ikeys(B, cap, g, n_valid=cap)
    qs = synth.decode_queries(B, seed=62)
    seq = torch.full((B,), 4 * cap, dtype=torch.int32)
    args = (synth.ikeys_swap_halves(ik).cuda(), isc.cuda(), seq.cuda(), 4, qs["q_idx"].cuda(), qs["head_w"].cuda(), k)
    ws = csld.indexer_workspace(B, cap, k)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    csld.lib.csld_test_set_barrier_extra(1)
    try:
        t0 = time.time()
        csld.indexer_topk(*args, ws=ws, err=err)
        torch.cuda.synchronize()
        waited = time.time() - t0
    finally:
        csld.lib.csld_test_set_barrier_extra(0)
    assert err.item() & CSLD_DEVERR_TIMEOUT, f"error word {err.item()}"
    assert waited < 30.0
    # the device is usable and a re-zeroed workspace gives the exact selection again
    ws.zero_()
    err.zero_()
    out = csld.indexer_topk(*args, ws=ws, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = orc.indexer_topk_batch(ik.numpy(), isc.numpy(), seq.numpy(), 4, qs["q_idx"].numpy(), qs["head_w"].numpy(), k)
    H.assert_topk_equal(out.cpu().numpy(), ref)
