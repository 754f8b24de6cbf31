"""ctypes binding of libkvq.so (the C ABI in include/kvq.h).

Argument marshalling only: every step of the cache and of decode attention
runs in the library's CUDA kernels. PyTorch supplies device memory (the cache
arena and the tensors passed in) and the current stream. If the shared library
is missing this module raises on import of the library: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = 0, -1, -2, -3, -4, -5
KVQ_F16, KVQ_BF16, KVQ_F32 = 0, 1, 2
KVQ_MAX_BATCH = 512

_DTYPE_CODE = {torch.float16: KVQ_F16, torch.bfloat16: KVQ_BF16, torch.float32: KVQ_F32}


class KvqError(RuntimeError):
    def __init__(self, status: int, func: str, detail: str):
        super().__init__(f"{func} failed with status {status}: {detail}")
        self.status = status


class kvq_config(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int32),
        ("max_batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("max_tokens", ctypes.c_int32),
        ("group_k", ctypes.c_int32),
        ("group_v", ctypes.c_int32),
        ("residual", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32),
        ("k_bits", ctypes.POINTER(ctypes.c_int8)),
        ("v_bits", ctypes.POINTER(ctypes.c_int8)),
        ("sink_tokens", ctypes.c_int32),
        ("k_axis", ctypes.POINTER(ctypes.c_int8)),
        ("hadamard", ctypes.c_int32),
        ("page_blocks", ctypes.c_int32),
        ("pool_pages", ctypes.c_int32),
        ("residual_v", ctypes.c_int32),
    ]


class kvq_layout(ctypes.Structure):
    _fields_ = [
        ("blocks", ctypes.c_void_p),
        ("record_bytes", ctypes.c_int64),
        ("max_blocks", ctypes.c_int64),
        ("kc_offset", ctypes.c_int64),
        ("ksz_offset", ctypes.c_int64),
        ("vc_offset", ctypes.c_int64),
        ("vsz_offset", ctypes.c_int64),
        ("ring_k", ctypes.c_void_p),
        ("ring_v", ctypes.c_void_p),
        ("k_bits", ctypes.c_int32),
        ("v_bits", ctypes.c_int32),
        ("sink_k", ctypes.c_void_p),
        ("sink_v", ctypes.c_void_p),
        ("k_axis", ctypes.c_int32),
        ("hadamard", ctypes.c_int32),
        ("page_table", ctypes.c_void_p),
        ("page_blocks", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("tile_tokens", ctypes.c_int32),
        ("tile_bytes", ctypes.c_int32),
        ("tile0_offset", ctypes.c_int32),
        ("rec_ksz_offset", ctypes.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkvq.so once and declare its signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m asymmetric_bit_kv_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    cfgp = ctypes.POINTER(kvq_config)
    sigs = {
        "kvq_cache_required_bytes": (I32, [cfgp, ctypes.POINTER(SZ)]),
        "kvq_cache_create": (I32, [cfgp, P, SZ, ctypes.POINTER(P)]),
        "kvq_cache_destroy": (I32, [P]),
        "kvq_cache_reset": (I32, [P, P]),
        "kvq_release_sequence": (I32, [P, I32, P]),
        "kvq_decode_attention_multi": (I32, [P, I32, P, P, I32, F32, I32, I32, P]),
        "kvq_append": (I32, [P, I32, P, P, ctypes.POINTER(I32), I32, P]),
        "kvq_flush_residual": (I32, [P, I32, I32, P]),
        "kvq_decode_attention": (I32, [P, I32, P, P, I32, F32, I32, P]),
        "kvq_decode_attention_noalloc": (I32, [P, I32, P, P, I32, F32, I32, P]),
        "kvq_decode_step": (I32, [P, I32, P, P, P, P, I32, F32, I32, P]),
        "kvq_dequant": (I32, [P, I32, I32, I32, I32, P, P, P]),
        "kvq_get_layout": (I32, [P, I32, ctypes.POINTER(kvq_layout)]),
        "kvq_device_errors": (I32, [P, ctypes.POINTER(I32)]),
        "kvq_cache_kernel_launches": (I32, [P, ctypes.POINTER(ctypes.c_uint64)]),
        "kvq_seq_lengths": (I32, [P, I32, I32, ctypes.POINTER(I32), ctypes.POINTER(I32)]),
        "kvq_seq_sinks": (I32, [P, I32, I32, ctypes.POINTER(I32)]),
        "kvq_seq_value_lengths": (I32, [P, I32, I32, ctypes.POINTER(I32), ctypes.POINTER(I32)]),
        "kvq_decode_kernel": (I32, [P, I32, I32, ctypes.POINTER(I32)]),
        "kvq_status_string": (ctypes.c_char_p, [I32]),
        "kvq_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(status: int, func: str):
    if status != KVQ_OK:
        lib = load_library()
        raise KvqError(status, func, lib.kvq_last_error().decode() or lib.kvq_status_string(status).decode())


def _stream_ptr(stream) -> int:
    """cudaStream_t of `stream`: a torch.cuda.Stream, a raw handle (int), or
    None for torch's current stream."""
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t: torch.Tensor, dtype, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclass
class CacheConfig:
    num_layers: int
    max_batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    max_tokens: int
    group_k: int
    group_v: int
    residual: int
    kv_dtype: torch.dtype
    k_bits: list
    v_bits: list
    sink_tokens: int = 0
    k_axis: list | None = None  # per layer: 0 keys per channel (KIVI), 1 per token (BQ2_0)
    hadamard: int = 0
    page_blocks: int = 0  # >= 1: block records in pages of this many blocks from a pool
    pool_pages: int = 0   # pages per layer (paged)
    residual_v: int = 0   # value ring slots when values keep their own window (0: residual)

    def to_c(self):
        kb = (ctypes.c_int8 * self.num_layers)(*self.k_bits)
        vb = (ctypes.c_int8 * self.num_layers)(*self.v_bits)
        ka = (ctypes.c_int8 * self.num_layers)(*(self.k_axis or [0] * self.num_layers))
        c = kvq_config(self.num_layers, self.max_batch, self.num_q_heads, self.num_kv_heads, self.head_dim,
                       self.max_tokens, self.group_k, self.group_v, self.residual, _DTYPE_CODE[self.kv_dtype],
                       ctypes.cast(kb, ctypes.POINTER(ctypes.c_int8)), ctypes.cast(vb, ctypes.POINTER(ctypes.c_int8)),
                       self.sink_tokens, ctypes.cast(ka, ctypes.POINTER(ctypes.c_int8)), self.hadamard,
                       self.page_blocks, self.pool_pages, self.residual_v)
        return c, (kb, vb, ka)


def required_bytes(cfg: CacheConfig) -> int:
    lib = load_library()
    c, _keep = cfg.to_c()
    n = ctypes.c_size_t(0)
    _check(lib.kvq_cache_required_bytes(ctypes.byref(c), ctypes.byref(n)), "kvq_cache_required_bytes")
    return n.value


def lens_array(new_lens) -> ctypes.Array:
    """new_lens as the int32 array kvq_append takes (reusable across calls)."""
    n = [int(x) for x in new_lens]
    return (ctypes.c_int32 * len(n))(*n)


class KVCache:
    """A packed KV cache bound to a torch-allocated device arena."""

    def __init__(self, cfg: CacheConfig, device="cuda"):
        self.lib = load_library()
        self.cfg = cfg
        self.device = torch.device(device)
        nbytes = required_bytes(cfg)
        with torch.cuda.device(self.device):
            self.arena = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            c, _keep = cfg.to_c()
            h = ctypes.c_void_p()
            _check(self.lib.kvq_cache_create(ctypes.byref(c), self.arena.data_ptr(), nbytes, ctypes.byref(h)),
                   "kvq_cache_create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            self.lib.kvq_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()

    def reset(self, stream=None):
        _check(self.lib.kvq_cache_reset(self.handle, _stream_ptr(stream)), "kvq_cache_reset")

    def release_sequence(self, seq: int, stream=None):
        """Empty sequence seq in every layer; a paged cache returns its pages
        (kvq_release_sequence)."""
        _check(self.lib.kvq_release_sequence(self.handle, seq, _stream_ptr(stream)), "kvq_release_sequence")

    def append(self, layer: int, k: torch.Tensor, v: torch.Tensor, new_lens, stream=None):
        """k, v: [sum(new_lens), Hkv, D] in the cache dtype; new_lens: ints per
        sequence (a list, or a ctypes int32 array from lens_array() to skip the
        per-call conversion)."""
        _need(k, self.cfg.kv_dtype, "k")
        _need(v, self.cfg.kv_dtype, "v")
        arr = new_lens if isinstance(new_lens, ctypes.Array) else lens_array(new_lens)
        _check(self.lib.kvq_append(self.handle, layer, k.data_ptr(), v.data_ptr(), arr, len(arr), _stream_ptr(stream)),
               "kvq_append")

    def flush_residual(self, layer: int, batch: int, stream=None):
        _check(self.lib.kvq_flush_residual(self.handle, layer, batch, _stream_ptr(stream)), "kvq_flush_residual")

    def decode_attention(self, layer: int, q: torch.Tensor, out: torch.Tensor | None = None,
                         out_dtype=torch.float32, softmax_scale: float | None = None, stream=None):
        """q: [batch, Hq, D] in the cache dtype. Returns out [batch, Hq, D]."""
        _need(q, self.cfg.kv_dtype, "q")
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        _need(out, out.dtype, "out")
        if softmax_scale is None:
            softmax_scale = self.cfg.head_dim ** -0.5
        _check(self.lib.kvq_decode_attention(self.handle, layer, q.data_ptr(), out.data_ptr(), _DTYPE_CODE[out.dtype],
                                             float(softmax_scale), q.shape[0], _stream_ptr(stream)),
               "kvq_decode_attention")
        return out

    def decode_step(self, layer: int, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                    out: torch.Tensor | None = None, out_dtype=torch.float32, softmax_scale: float | None = None,
                    stream=None):
        """Append one token per sequence (k, v: [batch, Hkv, D]) and decode
        (q: [batch, Hq, D]); kvq_decode_step. Returns out [batch, Hq, D]."""
        _need(k, self.cfg.kv_dtype, "k")
        _need(v, self.cfg.kv_dtype, "v")
        _need(q, self.cfg.kv_dtype, "q")
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        _need(out, out.dtype, "out")
        if softmax_scale is None:
            softmax_scale = self.cfg.head_dim ** -0.5
        _check(self.lib.kvq_decode_step(self.handle, layer, k.data_ptr(), v.data_ptr(), q.data_ptr(), out.data_ptr(),
                                        _DTYPE_CODE[out.dtype], float(softmax_scale), q.shape[0], _stream_ptr(stream)),
               "kvq_decode_step")
        return out

    def decode_attention_multi(self, layer: int, q: torch.Tensor, out_dtype=torch.float32,
                               softmax_scale: float | None = None, stream=None):
        """Several query tokens per sequence (q: [batch, T, Hq, D]), causal over
        the sequences' T newest tokens (kvq_decode_attention_multi). Returns
        out [batch, T, Hq, D]."""
        _need(q, self.cfg.kv_dtype, "q")
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        if softmax_scale is None:
            softmax_scale = self.cfg.head_dim ** -0.5
        _check(self.lib.kvq_decode_attention_multi(self.handle, layer, q.data_ptr(), out.data_ptr(),
                                                   _DTYPE_CODE[out.dtype], float(softmax_scale), q.shape[0],
                                                   q.shape[1], _stream_ptr(stream)),
               "kvq_decode_attention_multi")
        return out

    def decode_attention_noalloc(self, layer: int, q: torch.Tensor, out: torch.Tensor,
                                 softmax_scale: float | None = None, stream=None):
        """decode_attention with the split partials in the library's static
        device scratch instead of the arena (kvq_decode_attention_noalloc)."""
        _need(q, self.cfg.kv_dtype, "q")
        _need(out, out.dtype, "out")
        if softmax_scale is None:
            softmax_scale = self.cfg.head_dim ** -0.5
        _check(self.lib.kvq_decode_attention_noalloc(self.handle, layer, q.data_ptr(), out.data_ptr(),
                                                     _DTYPE_CODE[out.dtype], float(softmax_scale), q.shape[0],
                                                     _stream_ptr(stream)),
               "kvq_decode_attention_noalloc")
        return out

    def dequant(self, layer: int, seq: int, t0: int, t1: int, stream=None):
        """fp32 K_hat, V_hat [t1-t0, Hkv, D] of tokens [t0, t1) of one sequence."""
        shape = (t1 - t0, self.cfg.num_kv_heads, self.cfg.head_dim)
        k = torch.empty(shape, dtype=torch.float32, device=self.device)
        v = torch.empty(shape, dtype=torch.float32, device=self.device)
        _check(self.lib.kvq_dequant(self.handle, layer, seq, t0, t1, k.data_ptr(), v.data_ptr(), _stream_ptr(stream)),
               "kvq_dequant")
        return k, v

    def device_errors(self) -> int:
        """Device error flags since the last call (0 = none); synchronises."""
        f = ctypes.c_int32()
        _check(self.lib.kvq_device_errors(self.handle, ctypes.byref(f)), "kvq_device_errors")
        return f.value

    def kernel_launches(self) -> int:
        """Kernels enqueued so far by calls on this cache (kvq_cache_kernel_launches)."""
        n = ctypes.c_uint64()
        _check(self.lib.kvq_cache_kernel_launches(self.handle, ctypes.byref(n)), "kvq_cache_kernel_launches")
        return n.value

    def layout(self, layer: int) -> kvq_layout:
        lay = kvq_layout()
        _check(self.lib.kvq_get_layout(self.handle, layer, ctypes.byref(lay)), "kvq_get_layout")
        return lay

    def lengths(self, layer: int, seq: int):
        q = ctypes.c_int32()
        n = ctypes.c_int32()
        _check(self.lib.kvq_seq_lengths(self.handle, layer, seq, ctypes.byref(q), ctypes.byref(n)), "kvq_seq_lengths")
        return q.value, n.value

    def value_lengths(self, layer: int, seq: int):
        """(quantized values, value ring tokens) of one sequence (kvq_seq_value_lengths)."""
        q = ctypes.c_int32()
        n = ctypes.c_int32()
        _check(self.lib.kvq_seq_value_lengths(self.handle, layer, seq, ctypes.byref(q), ctypes.byref(n)),
               "kvq_seq_value_lengths")
        return q.value, n.value

    def decode_kernel(self, layer: int, rows_per_kv_head: int | None = None) -> str:
        """Decode kernel of a layer (kvq_decode_kernel): "cuda_core",
        "tensor_core" or "tensor_core_pair"; rows_per_kv_head defaults to one
        query token per sequence."""
        rows = rows_per_kv_head or self.cfg.num_q_heads // self.cfg.num_kv_heads
        k = ctypes.c_int32()
        _check(self.lib.kvq_decode_kernel(self.handle, layer, rows, ctypes.byref(k)), "kvq_decode_kernel")
        return ("cuda_core", "tensor_core", "tensor_core_pair")[k.value]

    def sinks(self, layer: int, seq: int) -> int:
        s = ctypes.c_int32()
        _check(self.lib.kvq_seq_sinks(self.handle, layer, seq, ctypes.byref(s)), "kvq_seq_sinks")
        return s.value
