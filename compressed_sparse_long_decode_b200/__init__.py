"""Python binding of libcsld.so -- the hybrid compressed-attention (CSA + HCA) decode path on
B200 (sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels behind the C ABI
declared in include/csld.h.  PyTorch provides device memory and streams.  There is no CPU
fallback: if the shared library is missing, importing this package raises.

Functions keep the C names (csa_compress, hca_compress, indexer_topk,
hybrid_decode_attention, kv_cache_append, kv_cache_prefill) and take torch tensors on the
current CUDA device; results are written into caller-provided tensors or freshly allocated
ones, on torch's current stream.
"""
import ctypes as C
import os

import torch

__all__ = [
    "csa_compress", "hca_compress", "compress", "compress_channel", "compress_rope", "kv_cache_append_rope",
    "kv_cache_prefill_rope", "compress_scaled", "kv_cache_append_scaled", "kv_cache_prefill_scaled",
    "hybrid_decode_attention_scaled", "compress_perhead", "kv_cache_prefill_perhead", "kv_cache_append_perhead",
    "indexer_topk_perhead", "indexer_topk", "hybrid_decode_attention",
    "kv_cache_append", "kv_cache_prefill", "LayerCache", "CsldError", "lib", "ENTRY_BYTES",
    "IKEY_BYTES", "DIM", "HEADS", "indexer_workspace", "attention_workspace", "DecodeStack",
    "layer_pattern", "stage", "indexer_rescore", "topk_merge", "lse_merge", "ContextParallelLayer",
    "partition_entries", "all_gather_stacked", "indexer_topk_multi", "indexer_multi_workspace",
    "hybrid_decode_attention_multi",
]

DIM = 512
DIM_NOPE = 448
ENTRY_BYTES = 576
IKEY_BYTES = 32
HEADS = 16
IDX_HEADS = 4
IDX_DIM = 64

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsld.so")


class CsldError(RuntimeError):
    pass


class _Cache(C.Structure):
    _fields_ = [
        ("ratio", C.c_int32), ("window", C.c_int32), ("batch", C.c_int32), ("has_indexer", C.c_int32),
        ("capacity", C.c_int64), ("comp_kv", C.c_void_p), ("ikeys", C.c_void_p),
        ("iscales", C.c_void_p), ("win_kv", C.c_void_p), ("tail_kv", C.c_void_p),
        ("tail_gate", C.c_void_p), ("seq_len", C.c_void_p), ("pos_bias", C.c_void_p),
        ("w_idx", C.c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libcsld.so not found at {LIB_PATH}; build it with "
                          "`python compressed_sparse_long_decode_b200/build.py`")
    L = C.CDLL(LIB_PATH)
    P, I, I64, F, S = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
    L.csld_abi_version.restype = I
    L.csld_last_error.restype = C.c_char_p
    L.csld_status_string.restype = C.c_char_p
    L.csld_status_string.argtypes = [I]
    L.csld_compress.argtypes = [P, P, P, I, P, I64, P, P, P, P]
    L.csld_compress_channel.argtypes = [P, P, P, I, P, I64, P, P, P, P]
    L.csld_compress_rope.argtypes = [P, P, P, I, P, I64, I64, C.c_double, P, P, P, P]
    L.kv_cache_append_rope.argtypes = [C.POINTER(_Cache), P, P, C.c_double, P, P]
    L.kv_cache_prefill_rope.argtypes = [C.POINTER(_Cache), P, P, I64, C.c_double, P]
    L.csld_compress_scaled.argtypes = [P, P, P, I, P, I64, F, P, P, P, P]
    L.kv_cache_append_scaled.argtypes = [C.POINTER(_Cache), P, P, F, P, P]
    L.kv_cache_prefill_scaled.argtypes = [C.POINTER(_Cache), P, P, I64, F, P]
    L.hybrid_decode_attention_scaled.argtypes = [P, I, P, I64, I, P, I, P, I, P, I, F, F, P, P, P, S, P, P]
    L.csld_compress_perhead.argtypes = [P, P, P, I, P, I64, P, P, P, P]
    L.kv_cache_prefill_perhead.argtypes = [C.POINTER(_Cache), P, P, I64, P]
    L.kv_cache_append_perhead.argtypes = [C.POINTER(_Cache), P, P, P, P]
    L.indexer_topk_perhead.argtypes = [P, P, I64, P, I, P, P, I, I, I, P, P, S, P, P]
    L.csa_compress.argtypes = [P, P, P, P, I64, P, P, P, P]
    L.hca_compress.argtypes = [P, P, P, I64, P, P]
    L.kv_cache_append.argtypes = [C.POINTER(_Cache), P, P, P, P]
    L.kv_cache_prefill.argtypes = [C.POINTER(_Cache), P, P, I64, P]
    L.csld_indexer_workspace_size.restype = S
    L.csld_indexer_workspace_size.argtypes = [I, I64, I]
    L.indexer_topk.argtypes = [P, P, I64, P, I, P, P, I, I, P, P, S, P, P]
    L.csld_attention_workspace_size.restype = S
    L.csld_attention_workspace_size.argtypes = [I, I, I64, I, I]
    L.hybrid_decode_attention.argtypes = [P, I, P, I64, I, P, I, P, I, P, I, F, P, P, P, S, P, P]
    L.csld_stage.argtypes = [P, P, S, P]
    L.indexer_rescore.argtypes = [P, P, I64, P, P, P, I, I, P, P]
    L.csld_indexer_multi_workspace_size.restype = S
    L.csld_indexer_multi_workspace_size.argtypes = [I, I, I64]
    L.indexer_topk_multi.argtypes = [P, P, I64, P, I, P, P, I, I, I, P, P, S, P, P]
    L.hybrid_decode_attention_multi.argtypes = [P, I, P, I64, I, P, I, P, I, I, P, I, I, F, P, P, P, S, P, P]
    L.csld_topk_merge.argtypes = [P, P, P, I, I, I, I64, I64, P, P]
    L.csld_lse_merge.argtypes = [P, P, I, I, I, P, P, P]
    for fn in ("csld_compress", "csld_compress_channel", "csld_compress_rope", "kv_cache_append_rope",
               "kv_cache_prefill_rope", "csld_compress_scaled", "kv_cache_append_scaled", "kv_cache_prefill_scaled",
               "hybrid_decode_attention_scaled", "csld_compress_perhead", "kv_cache_prefill_perhead",
               "kv_cache_append_perhead", "indexer_topk_perhead", "csa_compress", "hca_compress", "kv_cache_append", "kv_cache_prefill",
               "indexer_topk", "hybrid_decode_attention", "csld_stage", "indexer_rescore", "csld_topk_merge",
               "csld_lse_merge", "indexer_topk_multi", "hybrid_decode_attention_multi"):
        getattr(L, fn).restype = I
    return L


lib = _load()


def _check(status, what):
    if status != 0:
        msg = lib.csld_last_error().decode()
        raise CsldError(f"{what}: {lib.csld_status_string(status).decode()} ({msg})")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _need(t, dtype, name, host_ok=False):
    """t must be a contiguous tensor of dtype on the GPU, or (host_ok) in pinned host memory,
    which the kernels reach through unified addressing."""
    if t is None:
        raise CsldError(f"{name} is required")
    where_ok = t.is_cuda or (host_ok and t.is_pinned())
    if t.dtype != dtype or not where_ok or not t.is_contiguous():
        want = "CUDA or pinned host" if host_ok else "CUDA"
        raise CsldError(f"{name}: expected a contiguous {want} {dtype} tensor, got {t.dtype} "
                        f"{'cuda' if t.is_cuda else ('pinned cpu' if t.is_pinned() else 'cpu')} "
                        f"contiguous={t.is_contiguous()}")
    return t


def _bits(t, name):
    """bf16 tensor -> the same memory viewed as raw 16-bit patterns (no copy)."""
    _need(t, torch.bfloat16, name)
    return t


# ---- compression ------------------------------------------------------------------------
def compress(raw, gate, pos_bias, ratio, w_idx=None, kv_out=None, ikey_out=None, iscale_out=None):
    """Prefill compression of one sequence: raw [T,512] bf16, gate [T] f32, pos_bias [ratio]."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    _need(pos_bias, torch.float32, "pos_bias")
    T = raw.shape[0]
    E = T // ratio
    dev = raw.device
    if kv_out is None:
        kv_out = torch.empty((E, ENTRY_BYTES), dtype=torch.uint8, device=dev)
    if w_idx is not None:
        _need(w_idx, torch.float32, "w_idx")
        if ikey_out is None:
            ikey_out = torch.empty((E, IKEY_BYTES), dtype=torch.uint8, device=dev)
        if iscale_out is None:
            iscale_out = torch.empty((E, 2), dtype=torch.float32, device=dev)
    _check(lib.csld_compress(_ptr(raw), _ptr(gate), _ptr(pos_bias), ratio, _ptr(w_idx), T,
                             _ptr(kv_out), _ptr(ikey_out), _ptr(iscale_out), _stream()), "csld_compress")
    return (kv_out, ikey_out, iscale_out) if w_idx is not None else kv_out


def compress_channel(raw, gate, pos_bias, ratio, w_idx=None, kv_out=None, ikey_out=None, iscale_out=None):
    """Per-channel gated compression of one sequence: raw [T,512] bf16, gate [T,512] f32,
    pos_bias [ratio,512] f32 (csld_compress_channel)."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    _need(pos_bias, torch.float32, "pos_bias")
    T = raw.shape[0]
    E = T // ratio
    dev = raw.device
    if kv_out is None:
        kv_out = torch.empty((E, ENTRY_BYTES), dtype=torch.uint8, device=dev)
    if w_idx is not None:
        _need(w_idx, torch.float32, "w_idx")
        if ikey_out is None:
            ikey_out = torch.empty((E, IKEY_BYTES), dtype=torch.uint8, device=dev)
        if iscale_out is None:
            iscale_out = torch.empty((E, 2), dtype=torch.float32, device=dev)
    _check(lib.csld_compress_channel(_ptr(raw), _ptr(gate), _ptr(pos_bias), ratio, _ptr(w_idx), T, _ptr(kv_out),
                                     _ptr(ikey_out), _ptr(iscale_out), _stream()), "csld_compress_channel")
    return (kv_out, ikey_out, iscale_out) if w_idx is not None else kv_out


def compress_rope(raw, gate, pos_bias, ratio, pos0, rope_base, w_idx=None, kv_out=None, ikey_out=None,
                  iscale_out=None):
    """Compression with RoPE at compressed positions (csld_compress_rope): raw [T,512] bf16 with
    its dims 448..511 before rotary encoding, raw[0] at position pos0."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    _need(pos_bias, torch.float32, "pos_bias")
    T = raw.shape[0]
    E = T // ratio
    dev = raw.device
    if kv_out is None:
        kv_out = torch.empty((E, ENTRY_BYTES), dtype=torch.uint8, device=dev)
    if w_idx is not None:
        _need(w_idx, torch.float32, "w_idx")
        if ikey_out is None:
            ikey_out = torch.empty((E, IKEY_BYTES), dtype=torch.uint8, device=dev)
        if iscale_out is None:
            iscale_out = torch.empty((E, 2), dtype=torch.float32, device=dev)
    _check(lib.csld_compress_rope(_ptr(raw), _ptr(gate), _ptr(pos_bias), ratio, _ptr(w_idx), T, int(pos0),
                                  float(rope_base), _ptr(kv_out), _ptr(ikey_out), _ptr(iscale_out), _stream()),
           "csld_compress_rope")
    return (kv_out, ikey_out, iscale_out) if w_idx is not None else kv_out


def compress_scaled(raw, gate, pos_bias, ratio, kv_scale, w_idx=None, kv_out=None, ikey_out=None, iscale_out=None):
    """Compression into scaled FP8 entries (csld_compress_scaled)."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    _need(pos_bias, torch.float32, "pos_bias")
    T = raw.shape[0]
    E = T // ratio
    dev = raw.device
    if kv_out is None:
        kv_out = torch.empty((E, ENTRY_BYTES), dtype=torch.uint8, device=dev)
    if w_idx is not None:
        _need(w_idx, torch.float32, "w_idx")
        if ikey_out is None:
            ikey_out = torch.empty((E, IKEY_BYTES), dtype=torch.uint8, device=dev)
        if iscale_out is None:
            iscale_out = torch.empty((E, 2), dtype=torch.float32, device=dev)
    _check(lib.csld_compress_scaled(_ptr(raw), _ptr(gate), _ptr(pos_bias), ratio, _ptr(w_idx), T, float(kv_scale),
                                    _ptr(kv_out), _ptr(ikey_out), _ptr(iscale_out), _stream()), "csld_compress_scaled")
    return (kv_out, ikey_out, iscale_out) if w_idx is not None else kv_out


def compress_perhead(raw, gate, pos_bias, ratio, w_idx, kv_out=None, ikey_out=None, iscale_out=None):
    """Compression with per-head indexer keys (csld_compress_perhead): w_idx [512,4,64] f32 ->
    (kv [E,576], ikeys [E,128] in the stored layout, iscales [E,4,2])."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    _need(pos_bias, torch.float32, "pos_bias")
    _need(w_idx, torch.float32, "w_idx")
    T = raw.shape[0]
    E = T // ratio
    dev = raw.device
    if kv_out is None:
        kv_out = torch.empty((E, ENTRY_BYTES), dtype=torch.uint8, device=dev)
    if ikey_out is None:
        ikey_out = torch.empty((E, 4 * IKEY_BYTES), dtype=torch.uint8, device=dev)
    if iscale_out is None:
        iscale_out = torch.empty((E, 4, 2), dtype=torch.float32, device=dev)
    _check(lib.csld_compress_perhead(_ptr(raw), _ptr(gate), _ptr(pos_bias), ratio, _ptr(w_idx), T, _ptr(kv_out),
                                     _ptr(ikey_out), _ptr(iscale_out), _stream()), "csld_compress_perhead")
    return kv_out, ikey_out, iscale_out


def csa_compress(raw, gate, pos_bias, w_idx, kv_out=None, ikey_out=None, iscale_out=None):
    return compress(raw, gate, pos_bias, 4, w_idx, kv_out, ikey_out, iscale_out)


def hca_compress(raw, gate, pos_bias, kv_out=None):
    return compress(raw, gate, pos_bias, 128, None, kv_out)


# ---- cache state ------------------------------------------------------------------------
class LayerCache:
    """One layer's cache state for B sequences, in device memory owned by torch."""

    def __init__(self, batch, capacity, ratio, window, pos_bias, w_idx=None, device="cuda", perhead=False):
        """perhead: per-head indexer keys (w_idx [512,4,64]; ikeys [B,cap,128], iscales [B,cap,4,2]),
        filled by the *_perhead calls."""
        if w_idx is not None and capacity % 2:
            capacity += 1
        self.batch, self.capacity, self.ratio, self.window = batch, capacity, ratio, window
        dev = torch.device(device)
        self.comp_kv = torch.zeros((batch, capacity, ENTRY_BYTES), dtype=torch.uint8, device=dev)
        self.has_indexer = w_idx is not None
        self.perhead = perhead
        kshape = (batch, capacity, 4 * IKEY_BYTES) if perhead else (batch, capacity, IKEY_BYTES)
        sshape = (batch, capacity, 4, 2) if perhead else (batch, capacity, 2)
        self.ikeys = torch.zeros(kshape, dtype=torch.uint8, device=dev) if self.has_indexer else None
        self.iscales = torch.zeros(sshape, dtype=torch.float32, device=dev) if self.has_indexer else None
        self.win_kv = torch.zeros((batch, max(window, 1), ENTRY_BYTES), dtype=torch.uint8, device=dev)
        self.tail_kv = torch.zeros((batch, ratio, DIM), dtype=torch.bfloat16, device=dev)
        self.tail_gate = torch.zeros((batch, ratio), dtype=torch.float32, device=dev)
        self.seq_len = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.pos_bias = _need(pos_bias.to(dev).contiguous(), torch.float32, "pos_bias")
        self.w_idx = _need(w_idx.to(dev).contiguous(), torch.float32, "w_idx") if self.has_indexer else None
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def struct(self):
        return _Cache(self.ratio, self.window, self.batch, int(self.has_indexer), self.capacity,
                      _ptr(self.comp_kv), _ptr(self.ikeys), _ptr(self.iscales), _ptr(self.win_kv),
                      _ptr(self.tail_kv), _ptr(self.tail_gate), _ptr(self.seq_len),
                      _ptr(self.pos_bias), _ptr(self.w_idx))


def kv_cache_append(cache: LayerCache, kv_new, gate_new, err=None):
    """Append one token per sequence: kv_new [B,512] bf16, gate_new [B] f32."""
    _bits(kv_new, "kv_new")
    _need(gate_new, torch.float32, "gate_new")
    s = cache.struct()
    _check(lib.kv_cache_append(C.byref(s), _ptr(kv_new), _ptr(gate_new),
                               _ptr(cache.err if err is None else err), _stream()), "kv_cache_append")


def kv_cache_append_rope(cache: LayerCache, kv_new, gate_new, rope_base, err=None):
    """kv_cache_append with RoPE at compressed positions (kv_cache_append_rope)."""
    _bits(kv_new, "kv_new")
    _need(gate_new, torch.float32, "gate_new")
    s = cache.struct()
    _check(lib.kv_cache_append_rope(C.byref(s), _ptr(kv_new), _ptr(gate_new), float(rope_base),
                                    _ptr(cache.err if err is None else err), _stream()), "kv_cache_append_rope")


def kv_cache_prefill_rope(cache: LayerCache, raw, gate, rope_base):
    """kv_cache_prefill with RoPE at compressed positions (kv_cache_prefill_rope)."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    s = cache.struct()
    _check(lib.kv_cache_prefill_rope(C.byref(s), _ptr(raw), _ptr(gate), raw.shape[1], float(rope_base), _stream()),
           "kv_cache_prefill_rope")


def kv_cache_append_scaled(cache: LayerCache, kv_new, gate_new, kv_scale, err=None):
    """kv_cache_append into scaled FP8 entries (kv_cache_append_scaled)."""
    _bits(kv_new, "kv_new")
    _need(gate_new, torch.float32, "gate_new")
    s = cache.struct()
    _check(lib.kv_cache_append_scaled(C.byref(s), _ptr(kv_new), _ptr(gate_new), float(kv_scale),
                                      _ptr(cache.err if err is None else err), _stream()), "kv_cache_append_scaled")


def kv_cache_prefill_scaled(cache: LayerCache, raw, gate, kv_scale):
    """kv_cache_prefill into scaled FP8 entries (kv_cache_prefill_scaled)."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    s = cache.struct()
    _check(lib.kv_cache_prefill_scaled(C.byref(s), _ptr(raw), _ptr(gate), raw.shape[1], float(kv_scale), _stream()),
           "kv_cache_prefill_scaled")


def kv_cache_append_perhead(cache: LayerCache, kv_new, gate_new, err=None):
    """kv_cache_append with per-head indexer keys (kv_cache_append_perhead)."""
    _bits(kv_new, "kv_new")
    _need(gate_new, torch.float32, "gate_new")
    s = cache.struct()
    _check(lib.kv_cache_append_perhead(C.byref(s), _ptr(kv_new), _ptr(gate_new), _ptr(cache.err if err is None else err),
                                       _stream()), "kv_cache_append_perhead")


def kv_cache_prefill_perhead(cache: LayerCache, raw, gate):
    """kv_cache_prefill with per-head indexer keys (kv_cache_prefill_perhead)."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    s = cache.struct()
    _check(lib.kv_cache_prefill_perhead(C.byref(s), _ptr(raw), _ptr(gate), raw.shape[1], _stream()),
           "kv_cache_prefill_perhead")


def kv_cache_prefill(cache: LayerCache, raw, gate):
    """Prefill all sequences with T tokens: raw [B,T,512] bf16, gate [B,T] f32."""
    _bits(raw, "raw")
    _need(gate, torch.float32, "gate")
    s = cache.struct()
    _check(lib.kv_cache_prefill(C.byref(s), _ptr(raw), _ptr(gate), raw.shape[1], _stream()),
           "kv_cache_prefill")


# ---- indexer ------------------------------------------------------------------------------
def indexer_workspace(B, cap, k, device="cuda"):
    n = lib.csld_indexer_workspace_size(B, cap, k)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def indexer_topk(ikeys, iscales, seq_len, ratio, q_idx, head_w, k, out=None, ws=None, err=None):
    """ikeys [B,cap,32] u8, iscales [B,cap,2] f32, seq_len [B] i32, q_idx [B,4,64] f32,
    head_w [B,4] f32 -> top-k entry indices [B,k] i32 (ascending, -1 padded)."""
    _need(ikeys, torch.uint8, "ikeys")
    _need(iscales, torch.float32, "iscales")
    _need(seq_len, torch.int32, "seq_len")
    _need(q_idx, torch.float32, "q_idx")
    _need(head_w, torch.float32, "head_w")
    B, cap = ikeys.shape[0], ikeys.shape[1]
    if out is None:
        out = torch.empty((B, k), dtype=torch.int32, device=ikeys.device)
    if ws is None:
        ws = indexer_workspace(B, cap, k, ikeys.device)
    _check(lib.indexer_topk(_ptr(ikeys), _ptr(iscales), cap, _ptr(seq_len), ratio, _ptr(q_idx),
                            _ptr(head_w), B, k, _ptr(out), _ptr(ws), ws.numel(), _ptr(err), _stream()),
           "indexer_topk")
    return out


def indexer_multi_workspace(B, Q, cap, device="cuda"):
    n = lib.csld_indexer_multi_workspace_size(B, Q, cap)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def indexer_topk_perhead(ikeys, iscales, seq_len, ratio, q_idx, head_w, k, out=None, ws=None, err=None):
    """Per-head indexer keys (indexer_topk_perhead): ikeys [B,cap,128] u8 (stored layout),
    iscales [B,cap,4,2] f32, q_idx [B,Q,4,64] f32, head_w [B,Q,4] f32 -> top-k [B,Q,k] i32."""
    _need(ikeys, torch.uint8, "ikeys")
    _need(iscales, torch.float32, "iscales")
    _need(seq_len, torch.int32, "seq_len")
    _need(q_idx, torch.float32, "q_idx")
    _need(head_w, torch.float32, "head_w")
    B, cap = ikeys.shape[0], ikeys.shape[1]
    Q = q_idx.shape[1]
    if out is None:
        out = torch.empty((B, Q, k), dtype=torch.int32, device=ikeys.device)
    if ws is None:
        ws = indexer_multi_workspace(B, Q, cap, ikeys.device)
    _check(lib.indexer_topk_perhead(_ptr(ikeys), _ptr(iscales), cap, _ptr(seq_len), ratio, _ptr(q_idx), _ptr(head_w),
                                    B, Q, k, _ptr(out), _ptr(ws), ws.numel(), _ptr(err), _stream()),
           "indexer_topk_perhead")
    return out


def indexer_topk_multi(ikeys, iscales, seq_len, ratio, q_idx, head_w, k, out=None, ws=None, err=None):
    """Q query tokens per sequence in one pass over the keys: q_idx [B,Q,4,64] f32, head_w
    [B,Q,4] f32 -> top-k [B,Q,k] i32 (query j at raw position seq_len - Q + j)."""
    _need(ikeys, torch.uint8, "ikeys")
    _need(iscales, torch.float32, "iscales")
    _need(seq_len, torch.int32, "seq_len")
    _need(q_idx, torch.float32, "q_idx")
    _need(head_w, torch.float32, "head_w")
    B, cap = ikeys.shape[0], ikeys.shape[1]
    Q = q_idx.shape[1]
    if out is None:
        out = torch.empty((B, Q, k), dtype=torch.int32, device=ikeys.device)
    if ws is None:
        ws = indexer_multi_workspace(B, Q, cap, ikeys.device)
    _check(lib.indexer_topk_multi(_ptr(ikeys), _ptr(iscales), cap, _ptr(seq_len), ratio, _ptr(q_idx), _ptr(head_w),
                                  B, Q, k, _ptr(out), _ptr(ws), ws.numel(), _ptr(err), _stream()),
           "indexer_topk_multi")
    return out


# ---- attention ----------------------------------------------------------------------------
def attention_workspace(B, cap, k, W, device="cuda"):
    n = lib.csld_attention_workspace_size(B, HEADS, cap, k, W)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def hybrid_decode_attention(q, comp_kv, ratio, topk, win_kv, W, seq_len, scale, out=None,
                            lse=None, ws=None, err=None, kv_scale=None):
    """q [B,16,512] bf16; comp_kv [B,cap,576] u8; topk [B,k] i32 or None (dense); win_kv
    [B,W,576] u8; seq_len [B] i32 -> (out [B,16,512] f32, lse [B,16] f32).  kv_scale: scaled
    FP8 entries (hybrid_decode_attention_scaled); None for the base layout."""
    _bits(q, "q")
    _need(comp_kv, torch.uint8, "comp_kv")
    _need(seq_len, torch.int32, "seq_len")
    B, H = q.shape[0], q.shape[1]
    cap = comp_kv.shape[1]
    k = 0
    if topk is not None:
        _need(topk, torch.int32, "topk")
        k = topk.shape[1]
    if W > 0:
        _need(win_kv, torch.uint8, "win_kv")
    if out is None:
        out = torch.empty((B, H, DIM), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out", host_ok=True)   # a pinned host buffer receives the result directly
    if out.shape != (B, H, DIM):
        raise CsldError(f"out: expected shape {(B, H, DIM)}, got {tuple(out.shape)}")
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _need(lse, torch.float32, "lse", host_ok=True)
    if lse.shape != (B, H):
        raise CsldError(f"lse: expected shape {(B, H)}, got {tuple(lse.shape)}")
    if ws is None:
        ws = attention_workspace(B, cap, max(k, 1), W, q.device)
    if kv_scale is not None:
        _check(lib.hybrid_decode_attention_scaled(_ptr(q), H, _ptr(comp_kv), cap, ratio, _ptr(topk), k,
                                                  _ptr(win_kv) if W > 0 else None, W, _ptr(seq_len), B,
                                                  float(scale), float(kv_scale), _ptr(out), _ptr(lse), _ptr(ws),
                                                  ws.numel(), _ptr(err), _stream()), "hybrid_decode_attention_scaled")
        return out, lse
    _check(lib.hybrid_decode_attention(_ptr(q), H, _ptr(comp_kv), cap, ratio, _ptr(topk), k,
                                       _ptr(win_kv) if W > 0 else None, W, _ptr(seq_len), B,
                                       float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                       _ptr(err), _stream()), "hybrid_decode_attention")
    return out, lse


def hybrid_decode_attention_scaled(q, comp_kv, ratio, topk, win_kv, W, seq_len, scale, kv_scale, **kw):
    """hybrid_decode_attention over scaled FP8 entries (hybrid_decode_attention_scaled)."""
    return hybrid_decode_attention(q, comp_kv, ratio, topk, win_kv, W, seq_len, scale, kv_scale=kv_scale, **kw)


def hybrid_decode_attention_multi(q, comp_kv, ratio, topk, win_kv, W, seq_len, scale, out=None, lse=None, ws=None,
                                  err=None):
    """Q query tokens per sequence: q [B,Q,16,512] bf16; topk [B,Q,k] i32 or None; win_kv
    [B,W_ring,576] (W_ring >= W + Q - 1) -> (out [B,Q,16,512] f32, lse [B,Q,16] f32)."""
    _bits(q, "q")
    _need(comp_kv, torch.uint8, "comp_kv")
    _need(seq_len, torch.int32, "seq_len")
    B, Q, H = q.shape[0], q.shape[1], q.shape[2]
    cap = comp_kv.shape[1]
    k = 0
    if topk is not None:
        _need(topk, torch.int32, "topk")
        k = topk.shape[2]
    W_ring = win_kv.shape[1] if W > 0 else 0
    if W > 0:
        _need(win_kv, torch.uint8, "win_kv")
    if out is None:
        out = torch.empty((B, Q, H, DIM), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Q, H), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = attention_workspace(B * Q, cap, max(k, 1), W, q.device)
    _check(lib.hybrid_decode_attention_multi(_ptr(q), H, _ptr(comp_kv), cap, ratio, _ptr(topk), k,
                                             _ptr(win_kv) if W > 0 else None, W_ring, W, _ptr(seq_len), B, Q,
                                             float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _ptr(err),
                                             _stream()), "hybrid_decode_attention_multi")
    return out, lse


# ---- staging copies -----------------------------------------------------------------------
def stage(dst, src):
    """dst <- src (same byte size, both contiguous; each a CUDA tensor or pinned host memory)
    by a kernel on the current stream: csld_stage.  Returns dst."""
    for t, name in ((dst, "dst"), (src, "src")):
        if t is None or not t.is_contiguous() or not (t.is_cuda or t.is_pinned()):
            raise CsldError(f"{name}: expected a contiguous CUDA or pinned host tensor")
    nb = dst.numel() * dst.element_size()
    if src.numel() * src.element_size() != nb:
        raise CsldError("dst and src differ in size")
    _check(lib.csld_stage(_ptr(dst), _ptr(src), nb, _stream()), "csld_stage")
    return dst


# ---- a stack of layers --------------------------------------------------------------------
def layer_pattern(n_layers=61):
    """Layer kinds of the hybrid stack: layers 0 and 1 HCA, then CSA and HCA alternating from
    layer 2 (CSA) on -- for 61 layers, 30 CSA and 31 HCA ("DeepSeek-V4: a million-token context
    that agents can actually use", layer-pattern paragraph)."""
    return ["hca" if i < 2 or (i - 2) % 2 else "csa" for i in range(n_layers)]


class DecodeStack:
    """The attention layers of a hybrid stack for B sequences, each with its own cache (a
    LayerCache per layer), and one decode step through all of them: per layer kv_cache_append,
    then on CSA layers indexer_topk followed by sparse hybrid_decode_attention, on HCA layers
    dense hybrid_decode_attention.  The layers run in order on the current stream; every
    call is one of the C-ABI entry points above (this class only holds tensors).

    kinds: list of "csa" / "hca"; csa_cap / hca_cap: compressed-entry capacity per sequence;
    pos_bias4 [4], pos_bias128 [128], w_idx [512,64]: the pooling biases and the indexer
    projection (shared by the layers of a kind here; per-layer weights only change bytes)."""

    def __init__(self, batch, kinds, csa_cap, hca_cap, window, topk, pos_bias4, pos_bias128, w_idx,
                 device="cuda"):
        self.batch, self.kinds, self.window, self.topk = batch, list(kinds), window, topk
        dev = torch.device(device)
        self.layers = [LayerCache(batch, csa_cap, 4, window, pos_bias4, w_idx, device=dev) if k == "csa"
                       else LayerCache(batch, hca_cap, 128, window, pos_bias128, device=dev) for k in self.kinds]
        csa = [c for c in self.layers if c.ratio == 4]
        caps = [c.capacity for c in self.layers]
        self.ws_idx = indexer_workspace(batch, csa[0].capacity, topk, dev) if csa else None
        self.ws_att = attention_workspace(batch, max(caps), topk, window, dev)
        self.sel = torch.empty((batch, topk), dtype=torch.int32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def kv_bytes_per_sequence(self, context):
        """Bytes one sequence's cache holds at `context` raw tokens: compressed entries (576 B),
        indexer keys (32 B codes + 8 B scales) on CSA layers, the window ring and the tail."""
        total = 0
        for c in self.layers:
            n = context // c.ratio
            total += n * ENTRY_BYTES + (n * (IKEY_BYTES + 8) if c.has_indexer else 0)
            total += min(self.window, context) * ENTRY_BYTES + (context % c.ratio) * (2 * DIM + 4)
        return total

    def step(self, kv_new, gate_new, q, q_idx, head_w, scale, out, lse=None):
        """One decode token per sequence through every layer.  kv_new [L,B,512] bf16, gate_new
        [L,B] f32, q [L,B,16,512] bf16, q_idx [L,B,4,64] f32, head_w [L,B,4] f32; out
        [L,B,16,512] f32, lse [L,B,16] f32 or None (device tensors)."""
        for i, c in enumerate(self.layers):
            kv_cache_append(c, kv_new[i], gate_new[i], self.err)
            l_i = None if lse is None else lse[i]
            if c.has_indexer:
                indexer_topk(c.ikeys, c.iscales, c.seq_len, 4, q_idx[i], head_w[i], self.topk, out=self.sel,
                             ws=self.ws_idx, err=self.err)
                hybrid_decode_attention(q[i], c.comp_kv, 4, self.sel, c.win_kv, self.window, c.seq_len, scale,
                                        out=out[i], lse=l_i, ws=self.ws_att, err=self.err)
            else:
                hybrid_decode_attention(q[i], c.comp_kv, 128, None, c.win_kv, self.window, c.seq_len, scale,
                                        out=out[i], lse=l_i, ws=self.ws_att, err=self.err)


# ---- context-parallel split of a sequence over ranks -----------------------------------------
def indexer_rescore(ikeys, iscales, q_idx, head_w, sel, out=None):
    """fp32 scores [B,k] of the selected entries sel [B,k] (-inf where sel < 0): indexer_rescore."""
    for t, dt, n in ((ikeys, torch.uint8, "ikeys"), (iscales, torch.float32, "iscales"), (q_idx, torch.float32, "q_idx"),
                     (head_w, torch.float32, "head_w"), (sel, torch.int32, "sel")):
        _need(t, dt, n)
    B, k = sel.shape
    if out is None:
        out = torch.empty((B, k), dtype=torch.float32, device=sel.device)
    _need(out, torch.float32, "out")
    _check(lib.indexer_rescore(_ptr(ikeys), _ptr(iscales), ikeys.shape[1], _ptr(q_idx), _ptr(head_w), _ptr(sel), B, k,
                               _ptr(out), _stream()), "indexer_rescore")
    return out


def topk_merge(cand_scores, cand_idx, rank_lo, lo, n_local, out=None):
    """Global top-k over the gathered candidates cand_scores / cand_idx [R,B,k] (indices local to
    rank r's range starting at rank_lo[r], i64 [R] on the device), written as indices local to
    [lo, lo + n_local) (-1 elsewhere): csld_topk_merge."""
    _need(cand_scores, torch.float32, "cand_scores")
    _need(cand_idx, torch.int32, "cand_idx")
    _need(rank_lo, torch.int64, "rank_lo")
    R, B, k = cand_idx.shape
    if out is None:
        out = torch.empty((B, k), dtype=torch.int32, device=cand_idx.device)
    _need(out, torch.int32, "out")
    _check(lib.csld_topk_merge(_ptr(cand_scores), _ptr(cand_idx), _ptr(rank_lo), R, B, k, int(lo), int(n_local),
                               _ptr(out), _stream()), "csld_topk_merge")
    return out


def lse_merge(outs, lses, out=None, lse=None):
    """Combine partial attention results outs [R,B,16,512], lses [R,B,16]: csld_lse_merge."""
    _need(outs, torch.float32, "outs")
    _need(lses, torch.float32, "lses")
    R, B, H = lses.shape
    if out is None:
        out = torch.empty((B, H, DIM), dtype=torch.float32, device=outs.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=outs.device)
    _check(lib.csld_lse_merge(_ptr(outs), _ptr(lses), R, B, H, _ptr(out), _ptr(lse), _stream()), "csld_lse_merge")
    return out, lse


def all_gather_stacked(t, group=None):
    """[world, *t.shape]: every rank's t, in rank order (torch.distributed all-gather into one
    flat tensor: NCCL over NVLink between GPUs, gloo on CPU)."""
    import torch.distributed as td
    world = td.get_world_size(group)
    t = t.contiguous()
    flat = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    td.all_gather_into_tensor(flat, t, group=group)
    return flat.view((world,) + tuple(t.shape))


def partition_entries(n_entries, world):
    """Contiguous, near-equal ranges [lo_r, lo_r + n_r) of n_entries compressed entries over
    `world` ranks, each start a multiple of 8 (the key layout's 8-entry groups stay whole)."""
    per = -(-n_entries // world)
    per = -(-per // 8) * 8
    out = []
    for r in range(world):
        lo = min(n_entries, r * per)
        out.append((lo, min(n_entries, lo + per) - lo))
    return out


class ContextParallelLayer:
    """One layer's share of a context-parallel split on this rank: a LayerCache holding the
    compressed entries [lo, lo + n_local) of every sequence (indices local to the range), and, on
    the rank that owns the newest tokens, the window ring.  Lengths:
      cache.seq_len   ratio x the visible local entries (what indexer_topk and the local
                      attention see);
      seq_len_total   the sequence's raw tokens (the window branch; window rank only).
    step() runs one decode query through the layer on every rank of `group` (all ranks call it
    together): local indexer top-k and rescoring, an all-gather of the candidates, the exact
    global top-k, local attention, an all-gather of (out, lse), and their log-sum-exp merge.
    `all_gather(t)` returns the [R, ...] stack of every rank's t; the default uses
    torch.distributed (NCCL between GPUs)."""

    def __init__(self, cache: LayerCache, lo, n_local, rank_lo, window_rank, seq_len_total=None, group=None,
                 all_gather=None):
        self.cache, self.lo, self.n_local = cache, int(lo), int(n_local)
        self.rank_lo = rank_lo                      # i64 [R] on the device
        self.window_rank = bool(window_rank)
        self.seq_len_total = seq_len_total
        self.group = group
        self.all_gather = all_gather or self._dist_all_gather
        B = cache.batch
        dev = cache.comp_kv.device
        self._no_sel = torch.full((B, 1), -1, dtype=torch.int32, device=dev)

    def _dist_all_gather(self, t):
        import torch.distributed as td
        return all_gather_stacked(t, self.group)

    def step(self, q, scale, k=None, q_idx=None, head_w=None, ws_idx=None, ws_att=None, err=None):
        c = self.cache
        B = c.batch
        W = c.window if self.window_rank else 0
        parts_o, parts_l = [], []
        if c.has_indexer:
            sel = indexer_topk(c.ikeys, c.iscales, c.seq_len, c.ratio, q_idx, head_w, k, ws=ws_idx, err=err)
            sc = indexer_rescore(c.ikeys, c.iscales, q_idx, head_w, sel)
            g_sc, g_idx = self.all_gather(sc), self.all_gather(sel)
            mine = topk_merge(g_sc, g_idx, self.rank_lo, self.lo, self.n_local)
            seq = self.seq_len_total if self.window_rank else c.seq_len
            o, l = hybrid_decode_attention(q, c.comp_kv, c.ratio, mine, c.win_kv, W, seq, scale, ws=ws_att, err=err)
        else:
            o, l = hybrid_decode_attention(q, c.comp_kv, c.ratio, None, c.win_kv, 0, c.seq_len, scale, ws=ws_att,
                                           err=err)
            if self.window_rank and c.window > 0:
                # the window alone: a sparse call whose one selected slot is empty
                ow, lw = hybrid_decode_attention(q, c.comp_kv, c.ratio, self._no_sel, c.win_kv, c.window,
                                                 self.seq_len_total, scale, err=err)
                o, l = lse_merge(torch.stack([o, ow]), torch.stack([l, lw]))
        return lse_merge(self.all_gather(o), self.all_gather(l))
