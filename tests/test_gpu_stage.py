"""csld_stage (kernel copies between device memory and mapped pinned host memory) and attention
results written straight into pinned host memory."""
import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csld():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import compressed_sparse_long_decode_b200 as m
    return m


@pytest.mark.parametrize("nbytes", [16, 4096 + 48, 151552, 3 << 20])
def test_stage_host_to_device_to_host(csld, nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src = torch.randint(0, 256, (nbytes,), generator=g, dtype=torch.int32).to(torch.uint8).pin_memory()
    dev = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    back = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    csld.stage(dev, src)        # host -> device
    dev2 = torch.empty_like(dev)
    csld.stage(dev2, dev)       # device -> device
    csld.stage(back, dev2)      # device -> host
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu(), src)
    assert torch.equal(back, src)


def test_stage_refuses_misaligned_sizes(csld):
    a = torch.zeros(40, dtype=torch.uint8, device="cuda")
    b = torch.zeros(40, dtype=torch.uint8, device="cuda")
    with pytest.raises(csld.CsldError):
        csld.stage(a, b)        # 40 bytes: not a multiple of 16


def test_attention_writes_its_result_into_pinned_host_memory(csld):
    B, n, W = 4, 128 * 300, 128
    g = synth.gen(5)
    comp = synth.random_entries((B, n // 128 + 4), g)
    win = synth.random_entries((B, W), g)
    q = synth.decode_queries(B, seed=6)["q"].cuda()
    seq = torch.full((B,), n, dtype=torch.int32).cuda()
    scale = 1.0 / math.sqrt(512.0)
    o_dev, l_dev = csld.hybrid_decode_attention(q, comp.cuda(), 128, None, win.cuda(), W, seq, scale)
    o_host = torch.full((B, 16, 512), float("nan"), dtype=torch.float32).pin_memory()
    l_host = torch.full((B, 16), float("nan"), dtype=torch.float32).pin_memory()
    csld.hybrid_decode_attention(q, comp.cuda(), 128, None, win.cuda(), W, seq, scale, out=o_host, lse=l_host)
    torch.cuda.synchronize()
    assert np.array_equal(o_host.numpy(), o_dev.cpu().numpy())
    assert np.array_equal(l_host.numpy(), l_dev.cpu().numpy())
