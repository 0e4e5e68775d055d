"""Thin Python binding of ``libtq.so`` (argument marshalling only).

Every function mirrors the C entry point of the same name in ``include/tq.h``;
every step of the hot path runs in the library's CUDA kernels.  PyTorch is
used here only to allocate device memory and to hand over stream handles.
Importing this module loads the library and raises ``ImportError`` if it has
not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m kv_cache_vector_12_b200.build`")
lib = ctypes.CDLL(_LIB_PATH)

TQ_OK, TQ_ERR_INVALID, TQ_ERR_CUDA, TQ_ERR_NOMEM, TQ_ERR_UNSUPPORTED, TQ_ERR_DEVICE = range(6)
TQ_BF16, TQ_F32 = 0, 1
TQ_LAW_GAUSSIAN, TQ_LAW_SPHERE = 0, 1
LAWS = {"gaussian": TQ_LAW_GAUSSIAN, "sphere": TQ_LAW_SPHERE}
PLANES = ("codes_k", "norm_k", "qjl_bits", "qjl_norm", "codes_v", "norm_v")

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_fp = ctypes.POINTER(ctypes.c_float)


class tq_cache(ctypes.Structure):
    _fields_ = [("codes_k", _vp), ("norm_k", _vp), ("qjl_bits", _vp), ("qjl_norm", _vp),
                ("codes_v", _vp), ("norm_v", _vp), ("capacity", _i32), ("n_seqs", _i32),
                ("n_kv_heads", _i32), ("block_table", _vp), ("block_size", _i32), ("n_blocks", _i32)]


lib.tq_create.argtypes = [ctypes.POINTER(_vp), _i32, _i32, _i32, _i32, ctypes.c_uint64]
lib.tq_create.restype = ctypes.c_int
lib.tq_create_ex.argtypes = [ctypes.POINTER(_vp), _i32, _i32, _i32, _i32, ctypes.c_uint64, _i32]
lib.tq_create_ex.restype = ctypes.c_int
lib.tq_destroy.argtypes = [_vp]
lib.tq_destroy.restype = None
lib.tq_layout.argtypes = [_vp, ctypes.POINTER(ctypes.c_size_t)]
lib.tq_layout.restype = ctypes.c_int
lib.tq_get_params.argtypes = [_vp, _fp, _fp, _fp, _fp, _fp, _fp]
lib.tq_get_params.restype = ctypes.c_int
lib.tq_host_params.argtypes = [_i32, _i32, _i32, _i32, ctypes.c_uint64, _fp, _fp, _fp, _fp, _fp, _fp]
lib.tq_host_params.restype = ctypes.c_int
lib.tq_host_params_ex.argtypes = [_i32, _i32, _i32, _i32, ctypes.c_uint64, _i32, _fp, _fp, _fp, _fp, _fp, _fp]
lib.tq_host_params_ex.restype = ctypes.c_int
lib.tq_quantize.argtypes = [_vp, ctypes.POINTER(tq_cache), _vp, _vp, _vp, _vp, _i32, _vp]
lib.tq_quantize.restype = ctypes.c_int
lib.tq_workspace_bytes.argtypes = [_vp, _i32, _i32, _i32]
lib.tq_workspace_bytes.restype = ctypes.c_size_t
lib.tq_decode_attention.argtypes = [_vp, ctypes.POINTER(tq_cache), _vp, _i32, _i32, _vp, _i32,
                                    ctypes.c_float, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.tq_decode_attention.restype = ctypes.c_int
lib.tq_decode_attention_noalloc.argtypes = [_vp, ctypes.POINTER(tq_cache), _vp, _i32, _i32, _vp, _i32,
                                            ctypes.c_float, _vp, _vp, _vp]
lib.tq_decode_attention_noalloc.restype = ctypes.c_int
lib.tq_prefill_attention.argtypes = [_vp, ctypes.POINTER(tq_cache), _vp, _i32, _i32, _vp, _vp, _i32, _i32,
                                     ctypes.c_float, _vp, _vp, _vp]
lib.tq_prefill_attention.restype = ctypes.c_int
lib.tq_weight_quantize.argtypes = [_vp, ctypes.POINTER(tq_cache), _vp, _i32, _i32, _vp]
lib.tq_weight_quantize.restype = ctypes.c_int
lib.tq_weight_workspace_bytes.argtypes = [_vp, _i32, _i32]
lib.tq_weight_workspace_bytes.restype = ctypes.c_size_t
lib.tq_weight_gemm.argtypes = [_vp, ctypes.POINTER(tq_cache), _i32, _i32, _vp, _i32, _i32, _vp, _vp,
                               ctypes.c_size_t, _vp]
lib.tq_weight_gemm.restype = ctypes.c_int
lib.tq_check_device_errors.argtypes = [_vp, _vp]
lib.tq_check_device_errors.restype = ctypes.c_int
lib.tq_last_error.argtypes = []
lib.tq_last_error.restype = ctypes.c_char_p


class TQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"tq status {status}: {message}")
        self.status = status


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TQError(status, lib.tq_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _fbuf(t: torch.Tensor | None):
    return None if t is None else ctypes.cast(t.data_ptr(), _fp)


def _law(law) -> int:
    return LAWS[law] if isinstance(law, str) else int(law)


def host_params(d: int, bits_k: int, bits_v: int, qjl: int, seed: int, law="gaussian") -> dict:
    """tq_host_params_ex: the parameters tq_create_ex would upload (CPU only)."""
    out = {"pi": torch.empty(d * d), "s": torch.empty(d * d) if qjl else None,
           "centroids_k": torch.empty(1 << bits_k), "thresholds_k": torch.empty((1 << bits_k) - 1),
           "centroids_v": torch.empty(1 << bits_v), "thresholds_v": torch.empty((1 << bits_v) - 1)}
    _check(lib.tq_host_params_ex(d, bits_k, bits_v, qjl, seed, _law(law), _fbuf(out["pi"]), _fbuf(out["s"]),
                                 _fbuf(out["centroids_k"]), _fbuf(out["thresholds_k"]),
                                 _fbuf(out["centroids_v"]), _fbuf(out["thresholds_v"])))
    out["pi"] = out["pi"].view(d, d)
    if qjl:
        out["s"] = out["s"].view(d, d)
    return out


class Context:
    """Owns one tq_ctx (tq_create_ex / tq_destroy); law "gaussian" (the
    default, as tq_create) or "sphere" (tq_law)."""

    def __init__(self, d: int = 128, bits_k: int = 3, bits_v: int = 3, qjl: int = 0, seed: int = 42,
                 law="gaussian"):
        h = _vp()
        _check(lib.tq_create_ex(ctypes.byref(h), d, bits_k, bits_v, int(qjl), seed, _law(law)))
        self.handle = h
        self.d, self.bits_k, self.bits_v, self.qjl, self.seed = d, bits_k, bits_v, int(qjl), seed
        self.law = law

    def close(self) -> None:
        if self.handle:
            lib.tq_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layout(self) -> list[int]:
        arr = (ctypes.c_size_t * 6)()
        _check(lib.tq_layout(self.handle, arr))
        return list(arr)

    def params(self) -> dict:
        d = self.d
        out = {"pi": torch.empty(d * d), "s": torch.empty(d * d) if self.qjl else None,
               "centroids_k": torch.empty(1 << self.bits_k),
               "thresholds_k": torch.empty((1 << self.bits_k) - 1),
               "centroids_v": torch.empty(1 << self.bits_v),
               "thresholds_v": torch.empty((1 << self.bits_v) - 1)}
        _check(lib.tq_get_params(self.handle, _fbuf(out["pi"]), _fbuf(out["s"]),
                                 _fbuf(out["centroids_k"]), _fbuf(out["thresholds_k"]),
                                 _fbuf(out["centroids_v"]), _fbuf(out["thresholds_v"])))
        out["pi"] = out["pi"].view(d, d)
        if self.qjl:
            out["s"] = out["s"].view(d, d)
        return out

    def check_device_errors(self, stream=None) -> None:
        _check(lib.tq_check_device_errors(self.handle, _stream(stream)))


class Cache:
    """Device planes of one layer's packed cache, allocated through torch."""

    def __init__(self, ctx: Context, n_seqs: int, n_kv_heads: int, capacity: int, device="cuda"):
        sizes = ctx.layout()
        self.planes = {}
        for name, nbytes in zip(PLANES, sizes):
            if nbytes == 0:
                self.planes[name] = None
                continue
            shape = (n_seqs, n_kv_heads, capacity, nbytes) if nbytes > 2 else (n_seqs, n_kv_heads, capacity)
            dtype = torch.uint8 if nbytes > 2 else torch.int16
            self.planes[name] = torch.zeros(shape, dtype=dtype, device=device)
        self.n_seqs, self.n_kv_heads, self.capacity = n_seqs, n_kv_heads, capacity
        self.struct = tq_cache(*[_ptr(self.planes[n]) for n in PLANES], capacity, n_seqs, n_kv_heads, None, 0, 0)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.planes.values() if t is not None)


class PagedCache:
    """Device planes of one layer's packed cache in the paged layout:
    n_blocks physical blocks of block_size tokens ([n_blocks][n_kv_heads]
    [block_size][bytes] per plane) and a block table (device int32
    [n_seqs][capacity / block_size]) mapping each sequence's logical blocks
    to physical ones.  `block_table` may be given; by default sequence s owns
    physical blocks s * per_seq ... in order."""

    def __init__(self, ctx: Context, n_seqs: int, n_kv_heads: int, capacity: int, block_size: int,
                 n_blocks: int | None = None, block_table: torch.Tensor | None = None, device="cuda"):
        per_seq = capacity // block_size
        if n_blocks is None:
            n_blocks = n_seqs * per_seq
        if block_table is None:
            block_table = torch.arange(n_seqs * per_seq, dtype=torch.int32).view(n_seqs, per_seq)
        self.block_table = block_table.to(device=device, dtype=torch.int32).contiguous()
        sizes = ctx.layout()
        self.planes = {}
        for name, nbytes in zip(PLANES, sizes):
            if nbytes == 0:
                self.planes[name] = None
                continue
            shape = (n_blocks, n_kv_heads, block_size, nbytes) if nbytes > 2 else (n_blocks, n_kv_heads, block_size)
            dtype = torch.uint8 if nbytes > 2 else torch.int16
            self.planes[name] = torch.zeros(shape, dtype=dtype, device=device)
        self.n_seqs, self.n_kv_heads, self.capacity = n_seqs, n_kv_heads, capacity
        self.block_size, self.n_blocks = block_size, n_blocks
        self.struct = tq_cache(*[_ptr(self.planes[n]) for n in PLANES], capacity, n_seqs, n_kv_heads,
                               self.block_table.data_ptr(), block_size, n_blocks)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.planes.values() if t is not None)


def quantize(ctx: Context, cache: Cache, k: torch.Tensor, v: torch.Tensor, seq_idx: torch.Tensor,
             pos: torch.Tensor, stream=None) -> None:
    """tq_quantize: k, v bf16 [n_tok, n_kv_heads, d] contiguous; seq_idx, pos int32 [n_tok]."""
    n_tok = k.shape[0]
    _check(lib.tq_quantize(ctx.handle, ctypes.byref(cache.struct), _ptr(k), _ptr(v), _ptr(seq_idx),
                           _ptr(pos), n_tok, _stream(stream)))


def workspace_bytes(ctx: Context, n_seqs: int, n_q_heads: int, max_seq_len: int) -> int:
    return int(lib.tq_workspace_bytes(ctx.handle, n_seqs, n_q_heads, max_seq_len))


def decode_attention(ctx: Context, cache: Cache, q: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                     out: torch.Tensor, lse: torch.Tensor | None, workspace: torch.Tensor,
                     scale: float = 0.0, stream=None) -> None:
    """tq_decode_attention: q [n_seqs, n_q_heads, d] bf16 or fp32; out fp32 [n_seqs, n_q_heads, d]."""
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    n_q_heads = q.shape[1]
    _check(lib.tq_decode_attention(ctx.handle, ctypes.byref(cache.struct), _ptr(q), q_dtype, n_q_heads,
                                   _ptr(seq_lens), max_seq_len, scale, _ptr(out), _ptr(lse),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)))


def prefill_attention(ctx: Context, cache: Cache, q: torch.Tensor, cu_q: torch.Tensor, seq_lens: torch.Tensor,
                      max_q: int, max_seq_len: int, out: torch.Tensor, lse: torch.Tensor | None = None,
                      scale: float = 0.0, stream=None) -> None:
    """tq_prefill_attention: q [total, n_q_heads, d] bf16 or fp32, the queries of
    sequence s being rows cu_q[s]:cu_q[s+1] (its last positions below
    seq_lens[s], already quantized into the cache); out fp32 [total, n_q_heads, d]."""
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    _check(lib.tq_prefill_attention(ctx.handle, ctypes.byref(cache.struct), _ptr(q), q_dtype, q.shape[1],
                                    _ptr(cu_q), _ptr(seq_lens), max_q, max_seq_len, scale, _ptr(out), _ptr(lse),
                                    _stream(stream)))


def decode_attention_noalloc(ctx: Context, cache: Cache, q: torch.Tensor, seq_lens: torch.Tensor,
                             max_seq_len: int, out: torch.Tensor, lse: torch.Tensor | None,
                             scale: float = 0.0, stream=None) -> None:
    """tq_decode_attention_noalloc: decode attention without a caller workspace,
    for callers that cannot allocate device memory (the library's static
    scratch is used instead; concurrent calls on the GPU race on it)."""
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    _check(lib.tq_decode_attention_noalloc(ctx.handle, ctypes.byref(cache.struct), _ptr(q), q_dtype, q.shape[1],
                                           _ptr(seq_lens), max_seq_len, scale, _ptr(out), _ptr(lse),
                                           _stream(stream)))


class WeightCache:
    """Packed weight rows for tq_weight_quantize / tq_weight_gemm: a cache of
    one sequence whose KV heads are the n_in / d blocks of a row and whose
    positions are the n_out rows (K planes only)."""

    def __init__(self, ctx: Context, n_out: int, n_in: int, device="cuda"):
        nb = n_in // ctx.d
        cap = (n_out + 63) // 64 * 64
        sizes = ctx.layout()
        self.codes = torch.zeros((nb, cap, sizes[0]), dtype=torch.uint8, device=device)
        self.norms = torch.zeros((nb, cap), dtype=torch.int16, device=device)
        self.n_out, self.n_in, self.capacity = n_out, n_in, cap
        self.struct = tq_cache(self.codes.data_ptr(), self.norms.data_ptr(), None, None, None, None, cap, 1, nb,
                               None, 0, 0)

    def nbytes(self) -> int:
        return self.codes.numel() + 2 * self.norms.numel()


def weight_quantize(ctx: Context, wc: WeightCache, w: torch.Tensor, stream=None) -> None:
    """tq_weight_quantize: w bf16 [n_out, n_in] contiguous."""
    _check(lib.tq_weight_quantize(ctx.handle, ctypes.byref(wc.struct), _ptr(w), wc.n_out, wc.n_in, _stream(stream)))


def weight_workspace_bytes(ctx: Context, n_tok: int, n_in: int) -> int:
    return int(lib.tq_weight_workspace_bytes(ctx.handle, n_tok, n_in))


def weight_gemm(ctx: Context, wc: WeightCache, x: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                stream=None) -> None:
    """tq_weight_gemm: x [n_tok, n_in] bf16 or fp32; y fp32 [n_tok, n_out]."""
    x_dtype = TQ_F32 if x.dtype == torch.float32 else TQ_BF16
    _check(lib.tq_weight_gemm(ctx.handle, ctypes.byref(wc.struct), wc.n_out, wc.n_in, _ptr(x), x_dtype, x.shape[0],
                              _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)))


def alloc_workspace(ctx: Context, n_seqs: int, n_q_heads: int, max_seq_len: int, device="cuda") -> torch.Tensor:
    n = workspace_bytes(ctx, n_seqs, n_q_heads, max_seq_len)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)
