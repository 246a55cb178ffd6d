"""Host logic of the context-parallel split on CPU ranks over gloo (world size 2, 127.0.0.1):
the entry partition and the rank-ordered all-gather that carries the candidates and the partial
attention results between ranks.  The kernels themselves are covered by the GPU test
(tests/test_gpu_cp.py); the package is imported here without touching a device."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as td
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import compressed_sparse_long_decode_b200 as csld
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n = 1000
        parts = csld.partition_entries(n, world)
        lo, cnt = parts[rank]
        # every rank contributes (score, local index) candidates of its own range
        scores = torch.arange(cnt, dtype=torch.float32)[None, :3] + 100.0 * rank
        idx = torch.arange(3, dtype=torch.int32)[None, :]
        g_sc = csld.all_gather_stacked(scores)
        g_idx = csld.all_gather_stacked(idx)
        q.put((rank, parts, g_sc.tolist(), g_idx.tolist()))
        td.barrier()
    finally:
        td.destroy_process_group()


def test_partition_covers_every_entry_once():
    import compressed_sparse_long_decode_b200 as csld
    for n in (0, 1, 7, 8, 1000, 262144, 262147):
        for world in (1, 2, 3, 8):
            parts = csld.partition_entries(n, world)
            assert len(parts) == world
            covered = []
            for lo, cnt in parts:
                assert cnt >= 0 and lo % 8 == 0 or cnt == 0
                covered.extend(range(lo, lo + cnt))
            assert covered == list(range(n))


def test_all_gather_is_rank_ordered_on_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, parts, g_sc, g_idx in res:
        assert parts == [(0, 504), (504, 496)]
        assert g_sc == [[[0.0, 1.0, 2.0]], [[100.0, 101.0, 102.0]]]
        assert g_idx == [[[0, 1, 2]], [[0, 1, 2]]]
