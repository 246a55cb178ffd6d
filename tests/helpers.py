"""Comparison helpers shared by the GPU parity tests (tolerances as stated for the path).

- compressed entries: E4M3 codes within one code step of the float64 oracle's; bf16 RoPE
  values within one bf16 ulp of the oracle's plus the error bound of the GPU's fp32 weighted
  sum of m tokens, (m+2) 2^-24 max|x| (pool_slack) -- a value produced by cancellation near
  zero cannot be resolved to a bf16 ulp by an fp32 sum; the stated bar for the cache, one FP8
  ulp, is far looser than this;
- FP4 indexer keys: equal scales and codes within one grid step, except groups whose oracle
  amax/6 lies within 2^-8 (relative) of a power of two, where the scale may differ by one
  binade (the GPU forms the projection from bf16 operands);
- top-k sets: bit-exact; pairs of entries whose float64 scores differ by < 1e-6 relative are
  exempt when the float64 order is used;
- attention: |gpu - oracle| <= 2e-2 + 1e-2 |oracle| elementwise, for out and lse.
"""
import math

import numpy as np
import torch

ATOL = 2e-2
RTOL = 1e-2


def e4m3_ordinal(codes):
    c = np.asarray(codes).astype(np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def bf16_ordinal(bits):
    b = np.asarray(bits).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_values(bits):
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_ulp(vals):
    """Spacing of bf16 values at |vals| (the fp32 spacing times 2^16)."""
    return np.spacing(np.abs(vals).astype(np.float32)).astype(np.float64) * 65536.0


def pool_slack(raw_bf16, m):
    """fp32 error bound of an m-term convex combination of the given bf16 tokens."""
    x = np.abs(np.asarray(raw_bf16.float().cpu().numpy() if hasattr(raw_bf16, "float") else raw_bf16))
    return (m + 2) * 2.0 ** -24 * float(x.max(initial=0.0))


def entry_distance(gpu, ref):
    """(max E4M3 code distance, max bf16 |difference| in units of the oracle's ulp)."""
    gpu = np.asarray(gpu, np.uint8).reshape(-1, 576)
    ref = np.asarray(ref, np.uint8).reshape(-1, 576)
    d8 = np.abs(e4m3_ordinal(gpu[:, :448]) - e4m3_ordinal(ref[:, :448])).max(initial=0)
    g = bf16_values(gpu[:, 448:].copy().view(np.uint16))
    r = bf16_values(ref[:, 448:].copy().view(np.uint16))
    return int(d8), g, r


def assert_entries_close(gpu, ref, what="entries", abs_slack=0.0):
    d8, g, r = entry_distance(gpu, ref)
    assert d8 <= 1, f"{what}: E4M3 code distance {d8}"
    err = np.abs(g - r)
    bound = bf16_ulp(r) + abs_slack
    assert np.all(err <= bound), f"{what}: bf16 error {float((err - bound).max()):.3g} above bound"
    gb = np.asarray(gpu, np.uint8).reshape(-1)
    rb = np.asarray(ref, np.uint8).reshape(-1)
    return float((gb == rb).mean())


def _fp4_ord(codes):
    c = np.asarray(codes).astype(np.int32)
    return np.where(c & 8, -(c & 7), c & 7)


def unpack_fp4(keys):
    k = np.asarray(keys, np.uint8)
    lo = k & 0xF
    hi = k >> 4
    out = np.empty(k.shape[:-1] + (k.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def assert_fp4_keys_close(gkeys, gscales, rkeys, rscales, ramax=None):
    """gkeys/rkeys [E,32] u8, gscales/rscales [E,2] f32; ramax [E,2] oracle group amax (or None)."""
    gc = unpack_fp4(gkeys).reshape(-1, 2, 32)
    rc = unpack_fp4(rkeys).reshape(-1, 2, 32)
    gs = np.asarray(gscales, np.float32).reshape(-1, 2)
    rs = np.asarray(rscales, np.float32).reshape(-1, 2)
    same = gs == rs
    d = np.abs(_fp4_ord(gc) - _fp4_ord(rc)).max(axis=2)
    assert np.all(d[same] <= 1), f"FP4 codes differ by {d[same].max()} steps at equal scales"
    if not np.all(same):
        bad = np.argwhere(~same)
        assert ramax is not None, "scales differ and no oracle amax was given"
        for e, g in bad:
            ratio = gs[e, g] / rs[e, g]
            assert ratio in (0.5, 2.0), f"scale ratio {ratio}"
            a6 = float(ramax[e, g]) / 6.0
            near = abs(a6 / 2.0 ** round(math.log2(a6)) - 1.0) < 2.0 ** -8
            assert near, f"scales differ away from a power-of-two boundary (amax/6={a6})"
    return float(same.mean())


# Regression guard, tighter than the pass bar: the largest error must stay below 1 % of the
# largest output value (the arithmetic keeps about 2^-8 relative per product; measured errors
# are ~0.1 % of max |out|), so a precision regression in the kernel shows up even where the
# output is small next to ATOL.
GUARD = 1e-2


def assert_attention_close(gout, glse, rout, rlse, what="attention", guard=GUARD):
    gout = np.asarray(gout, np.float64)
    rout = np.asarray(rout, np.float64)
    err = np.abs(gout - rout)
    bound = ATOL + RTOL * np.abs(rout)
    worst = float((err - bound).max(initial=-1.0))
    assert np.all(err <= bound), f"{what}: out exceeds tolerance by {worst:.3g} (max abs err {err.max():.3g})"
    rmax = float(np.abs(rout).max(initial=0.0))
    assert float(err.max(initial=0.0)) <= guard * rmax, \
        f"{what}: max abs err {float(err.max(initial=0.0)):.3g} above {guard:g} x max|out| ({rmax:.3g})"
    if glse is not None:
        glse = np.asarray(glse, np.float64)
        rlse = np.asarray(rlse, np.float64)
        fin = np.isfinite(rlse)
        assert np.array_equal(np.isfinite(glse), fin), f"{what}: lse finiteness differs"
        le = np.abs(glse[fin] - rlse[fin])
        assert np.all(le <= ATOL + RTOL * np.abs(rlse[fin])), f"{what}: lse error {le.max():.3g}"
    return float(err.max(initial=0.0))


def assert_topk_equal(gpu, ref, score64=None):
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    assert gpu.shape == ref.shape
    if np.array_equal(gpu, ref):
        return
    bad = np.argwhere(np.any(gpu != ref, axis=-1)).ravel() if gpu.ndim == 2 else [None]
    raise AssertionError(f"top-k sets differ (rows {list(bad)[:8]})")


def near_tie_only(set_a, set_b, score64, rel=1e-6):
    """True if every entry in the symmetric difference of two selections has a partner on the
    other side whose float64 score is within rel of its own (the exemption for near-ties)."""
    a = set(int(x) for x in set_a if x >= 0)
    b = set(int(x) for x in set_b if x >= 0)
    only_a, only_b = a - b, b - a
    if not only_a and not only_b:
        return True
    if len(only_a) != len(only_b):
        return False
    sa = sorted(score64[i] for i in only_a)
    sb = sorted(score64[i] for i in only_b)
    return all(abs(x - y) <= rel * max(abs(x), abs(y), 1e-300) for x, y in zip(sa, sb))


def visible_entries(seq_len, ratio, cap):
    """Visible compressed entries of each sequence: min(seq_len / ratio, cap) (0 for seq_len < 0)."""
    n = np.asarray(seq_len, np.int64)
    return np.minimum(np.maximum(n, 0) // ratio, cap)


def assert_topk_matches_f64(orc, got, ikeys, iscales, seq_len, ratio, q_idx, head_w, k):
    """The stated top-k rule, checked on every sequence: the GPU set equals the selection made on
    the oracle's float64 scores (ties to the lower index), except for pairs of entries whose
    float64 scores differ by less than 1e-6 relative.  ikeys in the logical layout.  Returns the
    number of sequences on which that exemption was needed."""
    got = np.asarray(got)
    ikeys = np.asarray(ikeys)
    iscales = np.asarray(iscales)
    q_idx = np.asarray(q_idx, np.float32)
    head_w = np.asarray(head_w, np.float32)
    cap = ikeys.shape[1]
    n_vis = visible_entries(seq_len, ratio, cap)
    exempt = 0
    for b in range(got.shape[0]):
        n = int(n_vis[b])
        _, s64 = orc.indexer_scores(ikeys[b, :n], iscales[b, :n], q_idx[b], head_w[b])
        ref64 = orc.topk64(s64, k) if n > 0 else np.full(k, -1, np.int32)
        assert int((got[b] >= 0).sum()) == min(k, n), f"row {b}: {int((got[b] >= 0).sum())} entries, want {min(k, n)}"
        if not np.array_equal(np.sort(got[b][got[b] >= 0]), np.sort(ref64[ref64 >= 0])):
            assert near_tie_only(got[b], ref64, s64), f"row {b}: top-k differs from the float64 selection " \
                                                      f"beyond near-ties"
            exempt += 1
    return exempt


def planted_near_tie(n=2048, k=10, a=500, b=600):
    """Keys and a query on which the fp32 and the float64 orders differ at the top-k boundary.
    Head 0 reads group 0 of every key, head 1 group 1; head weights (1, 2^-30, 0, 0).  Nine
    entries score 384, entries a < b both have group 0 = 32 x 6.0 (score 192) and entry b also
    has group 1 = 32 x 0.5, which adds 2^-30 x 16 = 2^-26: below half an fp32 ulp of 192, so in
    fp32 the two tie and the lower index a wins, while in float64 b scores higher (relative
    difference 8e-11 < 1e-6: an exempt pair)."""
    ik = torch.zeros((1, n, 32), dtype=torch.uint8)
    isc = torch.ones((1, n, 2), dtype=torch.float32)
    big = list(range(100, 100 + k - 1))
    for i in big + [a, b]:
        ik[0, i, :16] = 0x77                      # group 0: every code 6.0
    isc[0, big, 0] = 2.0
    ik[0, b, 16:] = 0x11                          # group 1: every code 0.5
    q = torch.zeros((1, 4, 64))
    q[0, 0, :32] = 1.0
    q[0, 1, 32:] = 1.0
    w = torch.tensor([[1.0, 2.0 ** -30, 0.0, 0.0]])
    return ik, isc, q, w, big


def plant_aligned(comp, q, idx, g):
    """Overwrite entries idx[b] of comp [B,cap,576] with alpha * q[b, h] + N(0, 0.3^2) for a head h
    cycling over the 16 heads and alpha drawn from U(0.15, 0.6): each head then has a dozen or
    more entries whose logits stand 3-14 units above the rest, so its softmax is dominated by a
    few entries with distinct weights and distinct values (|out| ~ 0.3, far above the 2e-2
    absolute bar), unlike N(0,1) caches whose outputs are near-uniform averages."""
    B = comp.shape[0]
    qf = q.float()
    for b in range(B):
        n = len(idx[b])
        heads = torch.arange(n) % 16
        alpha = 0.15 + 0.45 * torch.rand(n, generator=g)
        x = alpha[:, None] * qf[b, heads] + 0.3 * torch.randn((n, 512), generator=g)
        comp[b, idx[b], :448] = x[:, :448].to(torch.float8_e4m3fn).view(torch.uint8)
        comp[b, idx[b], 448:] = x[:, 448:].to(torch.bfloat16).view(torch.uint8).reshape(n, 128)
