"""hybrid_decode_attention_static -- the attention entry point that allocates nothing.

Some callers cannot allocate device memory where they call the library: a plug-in whose host
framework owns every device allocation and passes it only inputs and outputs, or a decode
loop that must not enter the CUDA allocator between steps.  For them the library keeps one
fixed scratch array of its own.  This test drives that entry point through the C ABI
(ctypes on libcsld.so) and checks that, on two calls in a row, it returns what the regular
entry point with a caller workspace returns, within the attention tolerance the other tests
use, and what the float64 oracle returns.  It also checks that a call needing more scratch
than the array holds is refused before anything is launched.  It must pass on its own in a
fresh process as well as after the other tests (this file is collected last).
"""
import ctypes as C
import math
import os

import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "compressed_sparse_long_decode_b200", "libcsld.so")
P, I, I64, F, S = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L = C.CDLL(LIB)
    L.hybrid_decode_attention.argtypes = [P, I, P, I64, I, P, I, P, I, P, I, F, P, P, P, S, P, P]
    L.hybrid_decode_attention.restype = I
    L.hybrid_decode_attention_static.argtypes = [P, I, P, I64, I, P, I, P, I, P, I, F, P, P, P, P]
    L.hybrid_decode_attention_static.restype = I
    L.csld_attention_workspace_size.argtypes = [I, I, I64, I, I]
    L.csld_attention_workspace_size.restype = S
    L.csld_last_error.restype = C.c_char_p
    return L


def _ptr(t):
    return None if t is None else t.data_ptr()


def _case(B, cap, ratio, W, k, seed):
    g = synth.gen(seed)
    comp = synth.random_entries((B, cap), g).cuda()
    win = synth.random_entries((B, W), g).cuda()
    q = synth.decode_queries(B, seed=seed + 1)["q"].cuda()
    n = cap * ratio - 3
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    sel = None
    if k:
        n_vis = n // ratio
        sel = torch.stack([torch.sort(torch.randperm(n_vis, generator=g)[:k]).values for _ in range(B)])
        sel = sel.to(torch.int32).cuda()
    return comp, win, q, seq, sel


def _run_both(lib, comp, win, q, seq, sel, ratio, W):
    B, cap = comp.shape[0], comp.shape[1]
    k = 0 if sel is None else sel.shape[1]
    scale = 1.0 / math.sqrt(512.0)
    stream = torch.cuda.current_stream().cuda_stream
    out_ws = torch.empty((B, 16, 512), dtype=torch.float32, device="cuda")
    lse_ws = torch.empty((B, 16), dtype=torch.float32, device="cuda")
    nws = lib.csld_attention_workspace_size(B, 16, cap, max(k, 1), W)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    rc = lib.hybrid_decode_attention(_ptr(q), 16, _ptr(comp), cap, ratio, _ptr(sel), k, _ptr(win), W,
                                     _ptr(seq), B, scale, _ptr(out_ws), _ptr(lse_ws), _ptr(ws), nws, None, stream)
    assert rc == 0, lib.csld_last_error()
    out_st = torch.full((B, 16, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse_st = torch.full((B, 16), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.hybrid_decode_attention_static(_ptr(q), 16, _ptr(comp), cap, ratio, _ptr(sel), k, _ptr(win), W,
                                            _ptr(seq), B, scale, _ptr(out_st), _ptr(lse_st), _ptr(err), stream)
    assert rc == 0, lib.csld_last_error()
    torch.cuda.synchronize()
    assert err.item() == 0
    return out_ws.cpu().numpy(), lse_ws.cpu().numpy(), out_st.cpu().numpy(), lse_st.cpu().numpy()


def _oracle(orc, comp, win, q, seq, sel, ratio):
    return orc.attention_batch(synth.bits16(q.cpu()), comp.cpu().numpy(), ratio,
                               None if sel is None else sel.cpu().numpy(), win.cpu().numpy(), seq.cpu().numpy(),
                               1.0 / math.sqrt(512.0))


def test_static_scratch_matches_workspace_entry_point_twice(lib, orc):
    # first call: dense (HCA-like), 8 sequences
    comp, win, q, seq, _ = _case(8, 700, 128, 128, 0, seed=71)
    o1, l1, o2, l2 = _run_both(lib, comp, win, q, seq, None, 128, 128)
    H.assert_attention_close(o2, l2, o1, l1, "static scratch, first call (dense)")
    ro, rl = _oracle(orc, comp, win, q, seq, None, 128)
    H.assert_attention_close(o2, l2, ro, rl, "static scratch, first call (dense), against the oracle")
    # second call in a row reuses the same scratch: sparse (CSA-like), different shape
    comp, win, q, seq, sel = _case(3, 5000, 4, 64, 512, seed=72)
    o1, l1, o2, l2 = _run_both(lib, comp, win, q, seq, sel, 4, 64)
    H.assert_attention_close(o2, l2, o1, l1, "static scratch, second call (sparse)")
    ro, rl = _oracle(orc, comp, win, q, seq, sel, 4)
    H.assert_attention_close(o2, l2, ro, rl, "static scratch, second call (sparse), against the oracle")
    assert np.isfinite(o2).all()


def test_static_scratch_refuses_oversized_calls(lib):
    B, cap, W = 400, 64, 8       # 400 sequences need more scratch than the fixed array holds
    need = lib.csld_attention_workspace_size(B, 16, cap, 1, W)
    assert need > 8 * 1024 * 1024
    comp = torch.zeros((B, cap, 576), dtype=torch.uint8, device="cuda")
    win = torch.zeros((B, W, 576), dtype=torch.uint8, device="cuda")
    q = torch.zeros((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    seq = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, 16, 512), dtype=torch.float32, device="cuda")
    rc = lib.hybrid_decode_attention_static(_ptr(q), 16, _ptr(comp), cap, 4, None, 0, _ptr(win), W, _ptr(seq),
                                            B, 0.05, _ptr(out), None, None, torch.cuda.current_stream().cuda_stream)
    assert rc == 4                                       # CSLD_ERR_CAPACITY, nothing launched
    assert b"scratch" in lib.csld_last_error()
