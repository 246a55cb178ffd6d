"""GPU parity of the lightning indexer + top-k, at small sizes and at the full decode workloads,
including ties, padding and ragged lengths.  Every test checks two things on every sequence:
- the stated rule: the GPU set equals the selection on the oracle's float64 scores (ties to the
  lower index), except pairs of entries whose float64 scores differ by < 1e-6 relative;
- bit-exact equality with the oracle's fp32 selection (the fixed operation order both sides
  use to decide such near-ties)."""
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


def _run(csld, orc, ikeys, iscales, seq_len, q_idx, head_w, k, ratio=4):
    # the GPU reads the key cache's stored layout; the oracle the logical one
    dev = [t.cuda() for t in (synth.ikeys_swap_halves(ikeys), iscales, seq_len, q_idx, head_w)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = csld.indexer_topk(*dev[:3], ratio, dev[3], dev[4], k, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = orc.indexer_topk_batch(ikeys.numpy(), iscales.numpy(), seq_len.numpy(), ratio,
                                 q_idx.numpy(), head_w.numpy(), k)
    got = out.cpu().numpy()
    H.assert_topk_matches_f64(orc, got, ikeys.numpy(), iscales.numpy(), seq_len.numpy(), ratio,
                              q_idx.numpy(), head_w.numpy(), k)
    return got, ref


def _inputs(B, cap, n_valid, seed, heavy=0.0):
    g = synth.gen(seed)
    ik, isc = synth.random_ikeys(B, cap, g, heavy_frac=heavy, n_valid=n_valid)
    qs = synth.decode_queries(B, seed=seed + 1)
    return ik, isc, qs["q_idx"], qs["head_w"]


@pytest.mark.parametrize("B,n_c,k", [(1, 1024, 128), (3, 5000, 256), (2, 300, 512), (1, 8192 * 2 + 77, 1024),
                                     (4, 20000, 1), (2, 9000, 2048)])
def test_indexer_topk_matches_oracle(csld, orc, B, n_c, k):
    cap = n_c + (n_c & 1) + 64
    ik, isc, q, w = _inputs(B, cap, n_c, seed=B * 1000 + k)
    seq = torch.full((B,), 4 * n_c + 3, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)


def test_indexer_ragged_lengths_and_padding(csld, orc):
    B, cap, k = 6, 4096, 200
    ik, isc, q, w = _inputs(B, cap, cap, seed=5)
    seq = torch.tensor([0, 3, 4, 4 * 150 + 1, 4 * 4000, 4 * 5000], dtype=torch.int32)  # last: > cap
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)
    assert np.all(got[0] == -1) and np.all(got[1] == -1)
    assert got[2, 0] == 0 and np.all(got[2, 1:] == -1)
    assert np.array_equal(got[3, :150], np.arange(150)) and np.all(got[3, 150:] == -1)


def test_indexer_exact_ties_go_to_lower_index(csld, orc):
    B, cap, k = 2, 6000, 300
    ik = torch.zeros((B, cap, 32), dtype=torch.uint8)
    ik[:, :, :] = 0x22                                   # every code +1.0: identical keys
    ik[0, 4000:4100, :] = 0x44                           # 100 keys with code +2.0 on seq 0
    isc = torch.ones((B, cap, 2), dtype=torch.float32)
    q = torch.ones((B, 4, 64))
    w = torch.ones((B, 4))
    seq = torch.full((B,), 4 * cap, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)
    assert np.array_equal(got[1], np.arange(k))
    assert np.array_equal(got[0], np.concatenate([np.arange(200), np.arange(4000, 4100)]))


def test_indexer_negative_weights_and_relu(csld, orc):
    B, cap, k = 2, 2048, 64
    ik, isc, q, w = _inputs(B, cap, cap, seed=9)
    w[0] = torch.tensor([1.0, -2.0, 0.5, -0.25])
    w[1] = torch.tensor([-1.0, -1.0, -1.0, -1.0])       # all scores <= 0: ties at zero
    seq = torch.full((B,), 4 * cap, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)


@pytest.mark.parametrize("name", ["decode128k", "decode1m"])
def test_indexer_full_workloads(csld, orc, name):
    wl = synth.WORKLOADS[name]
    ik, isc, q, w = _inputs(wl.batch, wl.csa_cap, wl.csa_entries, seed=11, heavy=wl.heavy_frac)
    seq = torch.full((wl.batch,), wl.context, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, wl.topk)
    H.assert_topk_equal(got, ref)


@pytest.mark.parametrize("B,cap,k", [(300, 2048, 64), (40, 65536, 512)])
def test_indexer_many_sequences_merge_tree_path(csld, orc, B, cap, k):
    """Shapes whose CTAs cannot all be resident at once (more than 2 x 148 CTAs, or ranges
    longer than 8192 entries) take the merge-tree kernel instead of the cooperative one."""
    ik, isc, q, w = _inputs(B, cap, cap, seed=B + k)
    g = synth.gen(77)
    seq = (torch.randint(0, 4 * cap + 8, (B,), generator=g)).to(torch.int32)
    seq[0] = 4 * cap
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)


def test_indexer_workspace_reused_across_calls(csld, orc):
    """Each call clears the selection state the next call uses, so one zero-filled workspace
    serves any number of calls (here with different inputs; sequence 2 is short enough to skip
    the selection on calls 1 and 2, so its state sets alternate out of step with the others)."""
    B, cap, k = 4, 40000, 256
    ws = csld.indexer_workspace(B, cap, k)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for it in range(5):
        ik, isc, q, w = _inputs(B, cap, cap, seed=300 + it)
        short = 4 * 100 if it in (1, 2) else 4 * 1000
        seq = torch.tensor([4 * cap, 4 * (cap // 2) + 1, short, 4 * cap - 5], dtype=torch.int32)
        out = csld.indexer_topk(synth.ikeys_swap_halves(ik).cuda(), isc.cuda(), seq.cuda(), 4, q.cuda(), w.cuda(), k,
                                ws=ws, err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        ref = orc.indexer_topk_batch(ik.numpy(), isc.numpy(), seq.numpy(), 4, q.numpy(), w.numpy(), k)
        H.assert_topk_equal(out.cpu().numpy(), ref)
        H.assert_topk_matches_f64(orc, out.cpu().numpy(), ik.numpy(), isc.numpy(), seq.numpy(), 4, q.numpy(),
                                  w.numpy(), k)


def test_indexer_large_ties_take_the_slow_selection(csld, orc):
    """More than 8192 keys share the threshold's histogram bin (here: 40,000 identical keys
    with 300 larger ones planted), so the cooperative kernel resolves the threshold with two
    more histogram levels instead of its candidate list; ties still go to the lower indices."""
    B, cap, k = 2, 40000, 512
    ik = torch.full((B, cap, 32), 0x22, dtype=torch.uint8)     # every code +1.0: identical keys
    ik[0, 20000:20300, :] = 0x44                                # 300 keys with code +2.0 on seq 0
    isc = torch.ones((B, cap, 2), dtype=torch.float32)
    q = torch.ones((B, 4, 64))
    w = torch.ones((B, 4))
    seq = torch.full((B,), 4 * cap, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)
    assert np.array_equal(got[1], np.arange(k))
    assert np.array_equal(got[0], np.concatenate([np.arange(k - 300), np.arange(20000, 20300)]))


def test_indexer_threshold_bin_taken_whole(csld, orc):
    """The k-th largest key is the lowest key of its histogram bin, so the whole bin is taken
    and no key below it may be: on sequence 0 exactly k planted keys share the top bin, on
    sequence 1 the k planted keys have scales 2, 2, 4, 4, 8, ... (two per binade), and the
    other keys of the steps they sit in score lower; sequence 2 is random."""
    B, cap, k = 3, 6000, 100
    ik = torch.full((B, cap, 32), 0x22, dtype=torch.uint8)     # every code +1.0
    isc = torch.ones((B, cap, 2), dtype=torch.float32)
    ik[0, 4000:4000 + k, :] = 0x44                              # k keys with code +2.0
    planted = np.sort(np.random.default_rng(17).choice(cap, size=k, replace=False))
    for j, i in enumerate(planted):
        isc[1, int(i), :] = 2.0 ** (1 + j // 2)
    rk, rs, _, _ = _inputs(1, cap, cap, seed=23)
    ik[2], isc[2] = rk[0], rs[0]
    q = torch.ones((B, 4, 64))
    w = torch.ones((B, 4))
    seq = torch.full((B,), 4 * cap, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)
    assert np.array_equal(got[0], np.arange(4000, 4000 + k))
    assert np.array_equal(got[1], planted)


@pytest.mark.parametrize("ties", [False, True])
def test_indexer_one_long_sequence(csld, orc, ties):
    """One sequence of 262,144 entries split over 147 ranges (one CTA each): with random keys
    (1 % heavy) the threshold bin goes through the candidate list; with identical keys (300
    planted larger) it holds more than 8,192 keys and takes two more histogram levels."""
    B, n_c, k = 1, 262144, 1024
    if ties:
        ik = torch.full((B, n_c, 32), 0x22, dtype=torch.uint8)
        ik[0, 100000:100300, :] = 0x44
        isc = torch.ones((B, n_c, 2), dtype=torch.float32)
        q, w = torch.ones((B, 4, 64)), torch.ones((B, 4))
    else:
        ik, isc, q, w = _inputs(B, n_c, n_c, seed=41, heavy=0.01)
    seq = torch.full((B,), 4 * n_c, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)
    H.assert_topk_equal(got, ref)
    if ties:
        assert np.array_equal(got[0], np.concatenate([np.arange(k - 300), np.arange(100000, 100300)]))


def test_indexer_planted_near_tie_uses_the_exemption(csld, orc):
    n, k, a, b = 2048, 10, 500, 600
    ik, isc, q, w, big = H.planted_near_tie(n, k, a, b)
    seq = torch.full((1,), 4 * n, dtype=torch.int32)
    got, ref = _run(csld, orc, ik, isc, seq, q, w, k)     # includes the float64 rule on every row
    H.assert_topk_equal(got, ref)
    assert np.array_equal(got[0], np.array(sorted(big + [a]), np.int32))
    _, s64 = orc.indexer_scores(ik[0].numpy(), isc[0].numpy(), q[0].numpy(), w[0].numpy())
    ref64 = orc.topk64(s64, k)
    assert set(got[0]) ^ set(ref64) == {a, b}             # the exemption fired, for that pair only
