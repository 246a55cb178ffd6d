"""CPU oracle for the hybrid compressed-attention decode path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 implementation (``csld_oracle.c``) of what the CUDA library computes,
written from the pages about DeepSeek-V4 ("DeepSeek-V4: a million-token context that agents
can actually use": CSA / HCA paragraphs, Figures 3-4, storage paragraph; the velog.io paper
review: CSA, HCA and KV-cache-layout sections).  It shares no code with the CUDA path and
neither imports the other.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference leg may import it.

This module only marshals numpy arrays into the C functions; every step of the arithmetic is
in the C file.  ``parity unpinned``: the model's real gate form, indexer projection and FP4
scale rule (the pages give none); everything else is pinned by ``tests/test_oracle_pins.py``.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

ENTRY_BYTES = 576
D = 512
D_NOPE = 448
D_ROPE = 64
IDX_HEADS = 4
IDX_DIM = 64
IKEY_BYTES = 32

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = C.CDLL(path)
        _declare(_lib)
    return _lib


_P = C.c_void_p


def _declare(L):
    L.orc_e4m3_decode.restype = C.c_double
    L.orc_e4m3_decode.argtypes = [C.c_uint8]
    L.orc_e4m3_encode.restype = C.c_uint8
    L.orc_e4m3_encode.argtypes = [C.c_double]
    L.orc_bf16_decode.restype = C.c_double
    L.orc_bf16_decode.argtypes = [C.c_uint16]
    L.orc_bf16_encode.restype = C.c_uint16
    L.orc_bf16_encode.argtypes = [C.c_double]
    L.orc_e2m1_decode.restype = C.c_double
    L.orc_e2m1_decode.argtypes = [C.c_uint8]
    L.orc_e2m1_encode.restype = C.c_uint8
    L.orc_e2m1_encode.argtypes = [C.c_double]
    L.orc_fp4_group_scale.restype = C.c_double
    L.orc_fp4_group_scale.argtypes = [C.c_double]
    for name in ("orc_fp4_quantize64", "orc_fp4_dequantize64", "orc_entry_encode",
                 "orc_entry_decode", "orc_indexer_key_raw"):
        getattr(L, name).restype = None
    L.orc_fp4_quantize64.argtypes = [_P, _P, _P]
    L.orc_fp4_dequantize64.argtypes = [_P, _P, _P]
    L.orc_entry_encode.argtypes = [_P, _P]
    L.orc_entry_decode.argtypes = [_P, _P]
    L.orc_indexer_key_raw.argtypes = [_P, _P, _P]
    L.orc_pool_block.restype = None
    L.orc_pool_block.argtypes = [_P, _P, _P, C.c_int, _P]
    L.orc_compress.restype = None
    L.orc_compress.argtypes = [_P, _P, _P, _P, C.c_int64, C.c_int, _P, _P, _P]
    L.orc_rope_rotate.restype = None
    L.orc_rope_rotate.argtypes = [_P, C.c_double, C.c_double]
    L.orc_compress_rope.restype = None
    L.orc_compress_rope.argtypes = [_P, _P, _P, _P, C.c_int64, C.c_int, C.c_int64, C.c_double, _P, _P, _P]
    L.orc_pool_block_channel.restype = None
    L.orc_pool_block_channel.argtypes = [_P, _P, _P, C.c_int, _P]
    L.orc_compress_channel.restype = None
    L.orc_compress_channel.argtypes = [_P, _P, _P, _P, C.c_int64, C.c_int, _P, _P, _P]
    L.orc_indexer_scores.restype = None
    L.orc_indexer_scores.argtypes = [_P, _P, C.c_int64, _P, _P, _P, _P]
    L.orc_topk.restype = None
    L.orc_topk.argtypes = [_P, C.c_int64, C.c_int, _P]
    L.orc_topk64.restype = None
    L.orc_topk64.argtypes = [_P, C.c_int64, C.c_int, _P]
    L.orc_indexer_topk_batch.restype = None
    L.orc_indexer_topk_batch.argtypes = [_P, _P, C.c_int64, _P, C.c_int, _P, _P, C.c_int, C.c_int, _P]
    L.orc_attention.restype = C.c_int
    L.orc_attention.argtypes = [_P, C.c_int, _P, C.c_int64, C.c_int, _P, C.c_int, _P, C.c_int,
                                C.c_int32, C.c_double, _P, _P]
    L.orc_attention_batch.restype = C.c_int
    L.orc_attention_batch.argtypes = [_P, C.c_int, _P, C.c_int64, C.c_int, _P, C.c_int, _P, C.c_int,
                                      _P, C.c_int, C.c_double, _P, _P]
    L.orc_append.restype = C.c_int
    L.orc_append.argtypes = [C.c_int, C.c_int, C.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                             C.c_float]
    L.orc_append_batch.restype = C.c_int
    L.orc_append_batch.argtypes = [C.c_int, C.c_int, C.c_int64, C.c_int, _P, _P, _P, _P, _P, _P,
                                   _P, _P, _P, _P, _P]
    L.orc_append_batch_variant.restype = C.c_int
    L.orc_append_batch_variant.argtypes = [C.c_int, C.c_int, C.c_int64, C.c_int, _P, _P, _P, _P, _P, _P,
                                           _P, _P, _P, _P, _P, C.c_double, C.c_double, C.c_int]
    L.orc_indexer_key_raw_perhead.restype = None
    L.orc_indexer_key_raw_perhead.argtypes = [_P, _P, _P]
    L.orc_compress_perhead.restype = None
    L.orc_compress_perhead.argtypes = [_P, _P, _P, _P, C.c_int64, C.c_int, _P, _P, _P]
    L.orc_indexer_scores_perhead.restype = None
    L.orc_indexer_scores_perhead.argtypes = [_P, _P, C.c_int64, _P, _P, _P, _P]
    L.orc_indexer_topk_batch_perhead.restype = None
    L.orc_indexer_topk_batch_perhead.argtypes = [_P, _P, C.c_int64, _P, C.c_int, _P, _P, C.c_int, C.c_int, _P]
    L.orc_entry_encode_scaled.restype = None
    L.orc_entry_encode_scaled.argtypes = [_P, C.c_double, _P]
    L.orc_entry_decode_scaled.restype = None
    L.orc_entry_decode_scaled.argtypes = [_P, C.c_double, _P]
    L.orc_compress_scaled.restype = None
    L.orc_compress_scaled.argtypes = [_P, _P, _P, _P, C.c_int64, C.c_int, C.c_double, _P, _P, _P]
    L.orc_attention_batch_scaled.restype = C.c_int
    L.orc_attention_batch_scaled.argtypes = [_P, C.c_int, _P, C.c_int64, C.c_int, _P, C.c_int, _P, C.c_int,
                                             _P, C.c_int, C.c_double, C.c_double, _P, _P]
    L.orc_num_threads.restype = C.c_int
    L.orc_num_threads.argtypes = []


def _c(a, dtype):
    """Contiguous array of the exact dtype (no value conversion allowed)."""
    a = np.asarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def _ptr(a):
    return None if a is None else a.ctypes.data


# ---- codecs ------------------------------------------------------------------------------
def e4m3_decode(code):
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(x):
    return lib().orc_e4m3_encode(float(x))


def bf16_decode(bits):
    return lib().orc_bf16_decode(int(bits))


def bf16_encode(x):
    return lib().orc_bf16_encode(float(x))


def e2m1_decode(code):
    return lib().orc_e2m1_decode(int(code))


def e2m1_encode(v):
    return lib().orc_e2m1_encode(float(v))


def fp4_group_scale(amax):
    return lib().orc_fp4_group_scale(float(amax))


def fp4_quantize64(u):
    u = _c(u, np.float64)
    codes = np.zeros(IKEY_BYTES, np.uint8)
    scales = np.zeros(2, np.float32)
    lib().orc_fp4_quantize64(_ptr(u), _ptr(codes), _ptr(scales))
    return codes, scales


def fp4_dequantize64(codes, scales):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    out = np.zeros(IDX_DIM, np.float64)
    lib().orc_fp4_dequantize64(_ptr(codes), _ptr(scales), _ptr(out))
    return out


def entry_encode(x):
    x = _c(x, np.float64)
    e = np.zeros(ENTRY_BYTES, np.uint8)
    lib().orc_entry_encode(_ptr(x), _ptr(e))
    return e


def entry_decode(entry):
    entry = _c(entry, np.uint8)
    x = np.zeros(D, np.float64)
    lib().orc_entry_decode(_ptr(entry), _ptr(x))
    return x


def entries_decode(entries):
    entries = _c(entries, np.uint8).reshape(-1, ENTRY_BYTES)
    return np.stack([entry_decode(e) for e in entries]) if len(entries) else np.zeros((0, D))


# ---- O1 / O2 -----------------------------------------------------------------------------
def pool_block(raw_bits, gate, bias):
    """raw_bits: uint16 [m, 512] (bf16 bits); gate, bias: float32 [m] -> float64 [512]."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    m = raw_bits.shape[0]
    out = np.zeros(D, np.float64)
    lib().orc_pool_block(_ptr(raw_bits), _ptr(gate), _ptr(bias), m, _ptr(out))
    return out


def indexer_key_raw(c, w_idx):
    c = _c(c, np.float64)
    w_idx = _c(w_idx, np.float32)
    u = np.zeros(IDX_DIM, np.float64)
    lib().orc_indexer_key_raw(_ptr(c), _ptr(w_idx), _ptr(u))
    return u


def compress(raw_bits, gate, bias, m, w_idx=None):
    """Prefill compression of one sequence.  Returns (kv [E,576], ikeys [E,32], iscales [E,2])."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    T = raw_bits.shape[0]
    E = T // m
    kv = np.zeros((E, ENTRY_BYTES), np.uint8)
    ik = np.zeros((E, IKEY_BYTES), np.uint8) if w_idx is not None else None
    isc = np.zeros((E, 2), np.float32) if w_idx is not None else None
    w = _c(w_idx, np.float32) if w_idx is not None else None
    lib().orc_compress(_ptr(raw_bits), _ptr(gate), _ptr(bias), _ptr(w), T, m, _ptr(kv), _ptr(ik),
                       _ptr(isc))
    return kv, ik, isc


def rope_rotate(x, pos, base):
    """O1r: a copy of x (float64 [512]) with its RoPE dims 448..511 rotated at position pos."""
    x = np.array(x, dtype=np.float64, copy=True)
    assert x.shape == (D,)
    lib().orc_rope_rotate(_ptr(x), float(pos), float(base))
    return x


def compress_rope(raw_bits, gate, bias, m, pos0, base, w_idx=None):
    """Prefill compression with RoPE at compressed positions (raw token 0 at position pos0):
    entry s rotated at pos0 + (s+1) m - 1.  Returns (kv [E,576], ikeys [E,32], iscales [E,2])."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    T = raw_bits.shape[0]
    E = T // m
    kv = np.zeros((E, ENTRY_BYTES), np.uint8)
    ik = np.zeros((E, IKEY_BYTES), np.uint8) if w_idx is not None else None
    isc = np.zeros((E, 2), np.float32) if w_idx is not None else None
    w = _c(w_idx, np.float32) if w_idx is not None else None
    lib().orc_compress_rope(_ptr(raw_bits), _ptr(gate), _ptr(bias), _ptr(w), T, m, int(pos0), float(base),
                            _ptr(kv), _ptr(ik), _ptr(isc))
    return kv, ik, isc


def entry_encode_scaled(x, kv_scale):
    """Scaled FP8 entry: E4M3(x / kv_scale) for dims 0..447, bf16 for the RoPE dims."""
    x = _c(x, np.float64)
    e = np.zeros(ENTRY_BYTES, np.uint8)
    lib().orc_entry_encode_scaled(_ptr(x), float(kv_scale), _ptr(e))
    return e


def entry_decode_scaled(entry, kv_scale):
    entry = _c(entry, np.uint8)
    x = np.zeros(D, np.float64)
    lib().orc_entry_decode_scaled(_ptr(entry), float(kv_scale), _ptr(x))
    return x


def compress_scaled(raw_bits, gate, bias, m, kv_scale, w_idx=None):
    """Prefill compression into scaled FP8 entries.  Returns (kv [E,576], ikeys, iscales)."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    T = raw_bits.shape[0]
    E = T // m
    kv = np.zeros((E, ENTRY_BYTES), np.uint8)
    ik = np.zeros((E, IKEY_BYTES), np.uint8) if w_idx is not None else None
    isc = np.zeros((E, 2), np.float32) if w_idx is not None else None
    w = _c(w_idx, np.float32) if w_idx is not None else None
    lib().orc_compress_scaled(_ptr(raw_bits), _ptr(gate), _ptr(bias), _ptr(w), T, m, float(kv_scale), _ptr(kv),
                              _ptr(ik), _ptr(isc))
    return kv, ik, isc


def pool_block_channel(raw_bits, gate, bias):
    """Per-channel gating: raw_bits uint16 [m,512]; gate, bias float32 [m,512] -> float64 [512]."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    m = raw_bits.shape[0]
    out = np.zeros(D, np.float64)
    lib().orc_pool_block_channel(_ptr(raw_bits), _ptr(gate), _ptr(bias), m, _ptr(out))
    return out


def compress_channel(raw_bits, gate, bias, m, w_idx=None):
    """Per-channel prefill compression: gate [T,512], bias [m,512].  Returns (kv, ikeys, iscales)."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    T = raw_bits.shape[0]
    E = T // m
    kv = np.zeros((E, ENTRY_BYTES), np.uint8)
    ik = np.zeros((E, IKEY_BYTES), np.uint8) if w_idx is not None else None
    isc = np.zeros((E, 2), np.float32) if w_idx is not None else None
    w = _c(w_idx, np.float32) if w_idx is not None else None
    lib().orc_compress_channel(_ptr(raw_bits), _ptr(gate), _ptr(bias), _ptr(w), T, m, _ptr(kv), _ptr(ik), _ptr(isc))
    return kv, ik, isc


# ---- O3 / O4 -----------------------------------------------------------------------------
def indexer_scores(ikeys, iscales, q_idx, head_w):
    """ikeys [n,32] u8, iscales [n,2] f32, q_idx [4,64] f32, head_w [4] f32 -> (score32, score64)."""
    ikeys = _c(ikeys, np.uint8)
    iscales = _c(iscales, np.float32)
    q_idx = _c(q_idx, np.float32)
    head_w = _c(head_w, np.float32)
    n = ikeys.shape[0]
    s32 = np.zeros(max(n, 1), np.float32)
    s64 = np.zeros(max(n, 1), np.float64)
    lib().orc_indexer_scores(_ptr(ikeys), _ptr(iscales), n, _ptr(q_idx), _ptr(head_w), _ptr(s32),
                             _ptr(s64))
    return s32[:n], s64[:n]


def indexer_key_raw_perhead(c, w_idx):
    """Per-head keys before quantisation: c [512] f64, w_idx [512,4,64] f32 -> u [4,64] f64."""
    c = _c(c, np.float64)
    w_idx = _c(w_idx, np.float32)
    u = np.zeros((IDX_HEADS, IDX_DIM), np.float64)
    lib().orc_indexer_key_raw_perhead(_ptr(c), _ptr(w_idx), _ptr(u))
    return u


def compress_perhead(raw_bits, gate, bias, m, w_idx):
    """Prefill compression with per-head indexer keys (w_idx [512,4,64]).  Returns (kv [E,576],
    ikeys [E,4,32], iscales [E,4,2])."""
    raw_bits = _c(raw_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    w = _c(w_idx, np.float32)
    T = raw_bits.shape[0]
    E = T // m
    kv = np.zeros((E, ENTRY_BYTES), np.uint8)
    ik = np.zeros((E, IDX_HEADS, IKEY_BYTES), np.uint8)
    isc = np.zeros((E, IDX_HEADS, 2), np.float32)
    lib().orc_compress_perhead(_ptr(raw_bits), _ptr(gate), _ptr(bias), _ptr(w), T, m, _ptr(kv), _ptr(ik), _ptr(isc))
    return kv, ik, isc


def indexer_scores_perhead(ikeys, iscales, q_idx, head_w):
    """ikeys [n,4,32] u8, iscales [n,4,2] f32 (per-head keys), q_idx [4,64], head_w [4] ->
    (score32, score64)."""
    ikeys = _c(ikeys, np.uint8)
    iscales = _c(iscales, np.float32)
    q_idx = _c(q_idx, np.float32)
    head_w = _c(head_w, np.float32)
    n = ikeys.shape[0]
    s32 = np.zeros(max(n, 1), np.float32)
    s64 = np.zeros(max(n, 1), np.float64)
    lib().orc_indexer_scores_perhead(_ptr(ikeys), _ptr(iscales), n, _ptr(q_idx), _ptr(head_w), _ptr(s32),
                                     _ptr(s64))
    return s32[:n], s64[:n]


def indexer_topk_batch_perhead(ikeys, iscales, seq_len, ratio, q_idx, head_w, k):
    """ikeys [B,cap,4,32], iscales [B,cap,4,2] (per-head keys); the rest as indexer_topk_batch."""
    ikeys = _c(ikeys, np.uint8)
    iscales = _c(iscales, np.float32)
    seq_len = _c(seq_len, np.int32)
    q_idx = _c(q_idx, np.float32)
    head_w = _c(head_w, np.float32)
    B, cap = ikeys.shape[0], ikeys.shape[1]
    out = np.zeros((B, k), np.int32)
    lib().orc_indexer_topk_batch_perhead(_ptr(ikeys), _ptr(iscales), cap, _ptr(seq_len), ratio, _ptr(q_idx),
                                         _ptr(head_w), B, k, _ptr(out))
    return out


def topk(score32, k):
    score32 = _c(score32, np.float32)
    out = np.zeros(k, np.int32)
    lib().orc_topk(_ptr(score32), score32.shape[0], k, _ptr(out))
    return out


def topk64(score64, k):
    score64 = _c(score64, np.float64)
    out = np.zeros(k, np.int32)
    lib().orc_topk64(_ptr(score64), score64.shape[0], k, _ptr(out))
    return out


def indexer_topk_batch(ikeys, iscales, seq_len, ratio, q_idx, head_w, k):
    """ikeys [B,cap,32], iscales [B,cap,2], seq_len [B] i32, q_idx [B,4,64], head_w [B,4]."""
    ikeys = _c(ikeys, np.uint8)
    iscales = _c(iscales, np.float32)
    seq_len = _c(seq_len, np.int32)
    q_idx = _c(q_idx, np.float32)
    head_w = _c(head_w, np.float32)
    B, cap = ikeys.shape[0], ikeys.shape[1]
    out = np.zeros((B, k), np.int32)
    lib().orc_indexer_topk_batch(_ptr(ikeys), _ptr(iscales), cap, _ptr(seq_len), ratio, _ptr(q_idx),
                                 _ptr(head_w), B, k, _ptr(out))
    return out


# ---- O5 ----------------------------------------------------------------------------------
def attention_batch(q_bits, comp_kv, ratio, sel, win_kv, seq_len, scale, kv_scale=1.0):
    """q_bits [B,H,512] u16; comp_kv [B,cap,576]; sel [B,k] i32 or None; win_kv [B,W,576];
    seq_len [B] i32; kv_scale: scaled FP8 entries (1: the base layout).  Returns (out [B,H,512]
    f64, lse [B,H] f64)."""
    q_bits = _c(q_bits, np.uint16)
    comp_kv = _c(comp_kv, np.uint8)
    win_kv = _c(win_kv, np.uint8)
    seq_len = _c(seq_len, np.int32)
    B, H = q_bits.shape[0], q_bits.shape[1]
    cap = comp_kv.shape[1]
    W = win_kv.shape[1]
    k = 0
    if sel is not None:
        sel = _c(sel, np.int32)
        k = sel.shape[1]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    rc = lib().orc_attention_batch_scaled(_ptr(q_bits), H, _ptr(comp_kv), cap, ratio, _ptr(sel), k,
                                          _ptr(win_kv), W, _ptr(seq_len), B, float(scale), float(kv_scale),
                                          _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle attention: a selected index is not a visible entry")
    return out, lse


# ---- O6 ----------------------------------------------------------------------------------
class LayerState:
    """Host copy of one layer's cache state for B sequences (same layout as the device one)."""

    def __init__(self, B, cap, m, W, with_indexer, key_heads=1):
        self.B, self.cap, self.m, self.W = B, cap, m, W
        self.key_heads = key_heads
        self.comp_kv = np.zeros((B, cap, ENTRY_BYTES), np.uint8)
        kshape = (B, cap, IKEY_BYTES) if key_heads == 1 else (B, cap, key_heads, IKEY_BYTES)
        sshape = (B, cap, 2) if key_heads == 1 else (B, cap, key_heads, 2)
        self.ikeys = np.zeros(kshape, np.uint8) if with_indexer else None
        self.iscales = np.zeros(sshape, np.float32) if with_indexer else None
        self.win_kv = np.zeros((B, W, ENTRY_BYTES), np.uint8)
        self.tail_kv = np.zeros((B, m, D), np.uint16)
        self.tail_gate = np.zeros((B, m), np.float32)
        self.seq_len = np.zeros(B, np.int32)


def append_batch(st: LayerState, bias, w_idx, x_bits, gate, rope_base=0.0, kv_scale=1.0):
    """Append one token per sequence (x_bits [B,512] u16, gate [B] f32).  Raises on overflow.
    rope_base > 0: RoPE at compressed positions (window entry at its token, a completed entry
    at its block's last token); kv_scale: scaled FP8 entries (1: the base layout)."""
    bias = _c(bias, np.float32)
    w = _c(w_idx, np.float32) if w_idx is not None else None
    x_bits = _c(x_bits, np.uint16)
    gate = _c(gate, np.float32)
    rc = lib().orc_append_batch_variant(st.m, st.W, st.cap, st.B, _ptr(st.comp_kv), _ptr(st.ikeys),
                                        _ptr(st.iscales), _ptr(st.win_kv), _ptr(st.tail_kv),
                                        _ptr(st.tail_gate), _ptr(st.seq_len), _ptr(bias), _ptr(w),
                                        _ptr(x_bits), _ptr(gate), float(rope_base), float(kv_scale), st.key_heads)
    if rc != 0:
        raise OverflowError("oracle append: compressed cache capacity exceeded")


def num_threads():
    return lib().orc_num_threads()


def set_threads(n):
    os.environ["OMP_NUM_THREADS"] = str(n)
