"""Python binding of libkvq (include/kvq.h): argument marshalling only.

Every step of the hot path runs in the CUDA kernels behind the C ABI.  This
module loads ``libkvq.so`` with ctypes, turns torch CUDA tensors into raw
pointers and torch's current stream into a ``cudaStream_t``, and raises
``KVQError`` on any non-OK status.  There is no CPU fallback: if the library
is missing the import of the first call fails with a message saying so.
"""
from __future__ import annotations

import ctypes as C
import functools
import os
from dataclasses import dataclass

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# KVQ_LIBRARY may name another build of the same library (the bounds-checking
# libkvq_debug.so); the default is the release build next to this file
LIB_PATH = os.environ.get("KVQ_LIBRARY") or os.path.join(_PKG, "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = range(5)
KVQ_F32, KVQ_BF16 = 0, 1
# bytes of the fixed scratch array behind kvq_decode_attn_noalloc
# (KVQ_DECODE_NOALLOC_SCRATCH_BYTES in include/kvq.h)
KVQ_DECODE_NOALLOC_SCRATCH_BYTES = 8 << 20

EXPORTED = (
    "kvq_status_string", "kvq_version", "kvq_rotate", "kvq_quantize_append",
    "kvq_decode_attn_workspace", "kvq_decode_attn", "kvq_octave_layout_of",
    "kvq_octave_codebook", "kvq_octave_quantize", "kvq_octave_decode_attn_workspace",
    "kvq_octave_decode_attn", "kvq_decode_attn_noalloc", "kvq_decode_step",
    "kvq_decode_attn_multi", "kvq_device_errors", "kvq_set_wait_limit",
)
KVQ_DEVERR_WAIT_TIMEOUT, KVQ_DEVERR_BOUNDS = 1, 2


class KVQError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")
        self.status = status


class CacheDesc(C.Structure):
    _fields_ = [
        ("k_codes", C.c_void_p), ("k_scales", C.c_void_p),
        ("v_codes", C.c_void_p), ("v_scales", C.c_void_p),
        ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32),
        ("max_tokens", C.c_int32), ("batch_capacity", C.c_int32),
        ("block_table", C.c_void_p), ("page_size", C.c_int32),
        ("max_pages_per_seq", C.c_int32), ("num_pages", C.c_int32),
        ("code_bits", C.c_int32),
    ]


class OctaveFmtDesc(C.Structure):
    _fields_ = [("head_size", C.c_int32), ("rope_dim", C.c_int32),
                ("v_bits", C.c_int32), ("compact", C.c_int32)]


class OctaveLayoutDesc(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("off_k_nope", "off_v", "off_scales", "num_k_scales",
                                        "num_scales", "slot_bytes", "kernel_code")]


_lib = None


def lib():
    """Load libkvq.so (built by hadamard_rotated_bit_fwht_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m hadamard_rotated_bit_fwht_b200.build`")
        L = C.CDLL(LIB_PATH)
        L.kvq_status_string.restype = C.c_char_p
        L.kvq_status_string.argtypes = [C.c_int]
        L.kvq_version.restype = C.c_int
        L.kvq_rotate.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_int64, C.c_int32, C.c_void_p]
        L.kvq_quantize_append.argtypes = [C.POINTER(CacheDesc), C.c_void_p, C.c_void_p, C.c_int,
                                          C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]
        L.kvq_decode_attn_workspace.restype = C.c_size_t
        L.kvq_decode_attn_workspace.argtypes = [C.POINTER(CacheDesc), C.c_int32, C.c_int32,
                                                C.c_int32]
        L.kvq_decode_attn.argtypes = [C.POINTER(CacheDesc), C.c_void_p, C.c_int, C.c_int32,
                                      C.c_int32, C.c_void_p, C.c_int32, C.c_float, C.c_void_p,
                                      C.c_void_p, C.c_size_t, C.c_void_p]
        L.kvq_octave_layout_of.argtypes = [C.POINTER(OctaveFmtDesc), C.POINTER(OctaveLayoutDesc)]
        L.kvq_octave_codebook.argtypes = [C.c_int32, C.c_void_p, C.POINTER(C.c_float)]
        L.kvq_octave_quantize.argtypes = [C.POINTER(OctaveFmtDesc), C.c_void_p, C.c_void_p,
                                          C.c_int, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                          C.c_int32, C.c_int64, C.c_void_p, C.c_void_p]
        L.kvq_octave_decode_attn_workspace.restype = C.c_size_t
        L.kvq_octave_decode_attn_workspace.argtypes = [C.POINTER(OctaveFmtDesc), C.c_int32,
                                                       C.c_int32, C.c_int32]
        L.kvq_octave_decode_attn.argtypes = [
            C.POINTER(OctaveFmtDesc), C.c_void_p, C.c_int, C.c_int32, C.c_int32, C.c_void_p,
            C.c_int32, C.c_int32, C.c_int64, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p,
            C.c_void_p, C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
            C.c_void_p]
        L.kvq_decode_attn_noalloc.argtypes = [C.POINTER(CacheDesc), C.c_void_p, C.c_int, C.c_int32,
                                              C.c_int32, C.c_void_p, C.c_int32, C.c_float,
                                              C.c_void_p, C.c_void_p]
        L.kvq_decode_attn_multi.argtypes = [C.POINTER(CacheDesc), C.c_void_p, C.c_int, C.c_int32,
                                            C.c_int32, C.c_void_p, C.c_void_p, C.c_int32,
                                            C.c_int32, C.c_float, C.c_void_p, C.c_void_p,
                                            C.c_size_t, C.c_void_p]
        L.kvq_decode_step.argtypes = [C.POINTER(CacheDesc), C.c_void_p, C.c_void_p, C.c_void_p,
                                      C.c_int, C.c_int32, C.c_int32, C.c_void_p, C.c_int32,
                                      C.c_float, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
        L.kvq_device_errors.argtypes = [C.POINTER(C.c_uint32)]
        L.kvq_set_wait_limit.argtypes = [C.c_int32]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kvq_status_string(status).decode()


def _check(fn, status):
    if status != KVQ_OK:
        raise KVQError(fn, status)


# the raw handle of torch's current stream on the current device, without
# building a Stream object (this sits on the per-token decode path); the
# public route where this torch build lacks the internal accessor
_RAW_STREAM = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream=None):
    if stream is not None:
        return stream.cuda_stream
    if _RAW_STREAM is not None:
        return _RAW_STREAM(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KVQ_F32
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    raise TypeError(f"expected float32 or bfloat16, got {t.dtype}")


def _cuda_contig(name, t):
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


# --------------------------------------------------------------------------
# Q4_0 + FWHT-256
# --------------------------------------------------------------------------
class Q4Cache:
    """Caller-owned structure-of-arrays Q4_0 (bits=4) or Q8_0 (bits=8) cache
    (layout in include/kvq.h)."""

    def __init__(self, n_rows, num_kv_heads, device, *, max_tokens=0, batch_capacity=0,
                 block_table=None, page_size=0, num_pages=0, bits=4):
        if bits not in (4, 8):
            raise ValueError("bits must be 4 (Q4_0) or 8 (Q8_0)")
        dev = torch.device(device)
        self.bits = bits
        self.num_kv_heads = num_kv_heads
        self.max_tokens = max_tokens
        self.batch_capacity = batch_capacity
        self.block_table = block_table
        self.page_size = page_size
        self.num_pages = num_pages
        self.k_codes = torch.zeros((n_rows, 32 * bits), dtype=torch.uint8, device=dev)
        self.v_codes = torch.zeros((n_rows, 32 * bits), dtype=torch.uint8, device=dev)
        self.k_scales = torch.zeros((n_rows, 8), dtype=torch.int16, device=dev)
        self.v_scales = torch.zeros((n_rows, 8), dtype=torch.int16, device=dev)

    @classmethod
    def contiguous(cls, batch, num_kv_heads, max_tokens, device="cuda", bits=4):
        return cls(batch * num_kv_heads * max_tokens, num_kv_heads, device,
                   max_tokens=max_tokens, batch_capacity=batch, bits=bits)

    @classmethod
    def paged(cls, num_pages, num_kv_heads, page_size, block_table, device="cuda", bits=4):
        bt = block_table.to(device=device, dtype=torch.int32).contiguous()
        return cls(num_pages * num_kv_heads * page_size, num_kv_heads, device,
                   block_table=bt, page_size=page_size, num_pages=num_pages, bits=bits)

    def with_block_table(self, block_table: torch.Tensor) -> "Q4Cache":
        """The same planes seen through another block table (e.g. one row, to
        append a single sequence of a paged batch)."""
        view = Q4Cache.__new__(Q4Cache)
        view.__dict__.update(self.__dict__)
        view.__dict__.pop("_desc", None)
        view.block_table = block_table.to(device=self.k_codes.device,
                                          dtype=torch.int32).contiguous()
        return view

    @property
    def capacity(self):
        if self.block_table is None:
            return self.max_tokens
        return self.block_table.shape[1] * self.page_size

    def desc(self) -> CacheDesc:
        """The C descriptor, built once (the planes and the block table of a
        Q4Cache object never change; with_block_table makes a new object)."""
        d = self.__dict__.get("_desc")
        if d is None:
            bt = self.block_table
            d = CacheDesc(self.k_codes.data_ptr(), self.k_scales.data_ptr(),
                          self.v_codes.data_ptr(), self.v_scales.data_ptr(),
                          self.num_kv_heads, 256, self.max_tokens, self.batch_capacity,
                          None if bt is None else bt.data_ptr(), self.page_size,
                          0 if bt is None else bt.shape[1], self.num_pages, self.bits)
            self._desc = d
        return d

    def nbytes_per_row(self):
        return 2 * (32 * self.bits + 16)


def rotate(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = H x over the last dim (256), fp32 output."""
    _cuda_contig("x", x)
    if x.shape[-1] != 256:
        raise ValueError("kvq_rotate: last dim must be 256")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    n = x.numel() // 256
    _check("kvq_rotate", lib().kvq_rotate(_ptr(x), _dtype_code(x), _ptr(out), n, 256,
                                          _stream(stream)))
    return out


def quantize_append(cache: Q4Cache, k: torch.Tensor, v: torch.Tensor,
                    start_pos: torch.Tensor, stream=None) -> None:
    """Rotate + Q4_0-quantize k, v ([batch, t_new, Hkv, 256]) into the cache."""
    _cuda_contig("k", k)
    _cuda_contig("v", v)
    _cuda_contig("start_pos", start_pos)
    if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4:
        raise ValueError("k and v must have the same [batch, t_new, Hkv, 256] shape and dtype")
    if start_pos.dtype != torch.int32:
        raise TypeError("start_pos must be int32")
    batch, t_new, hkv, _ = k.shape
    if hkv != cache.num_kv_heads:
        raise ValueError("kv head count does not match the cache")
    d = cache.desc()
    _check("kvq_quantize_append",
           lib().kvq_quantize_append(C.byref(d), _ptr(k), _ptr(v), _dtype_code(k), batch, t_new,
                                     _ptr(start_pos), _stream(stream)))


def decode_attn_workspace(cache: Q4Cache, batch: int, num_q_heads: int, max_seq_len: int) -> int:
    d = cache.desc()
    return int(lib().kvq_decode_attn_workspace(C.byref(d), batch, num_q_heads, max_seq_len))


def decode_attn(cache: Q4Cache, q: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                scale: float, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One query token per sequence: q [batch, Hq, 256] -> out [batch, Hq, 256] fp32."""
    _cuda_contig("q", q)
    _cuda_contig("seq_lens", seq_lens)
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    batch, hq, dim = q.shape
    if out is None:
        out = torch.empty((batch, hq, dim), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_attn_workspace(cache, batch, hq, max_seq_len)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    d = cache.desc()
    _check("kvq_decode_attn",
           lib().kvq_decode_attn(C.byref(d), _ptr(q), _dtype_code(q), batch, hq, _ptr(seq_lens),
                                 int(max_seq_len), float(scale), _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def decode_attn_multi(cache: Q4Cache, q: torch.Tensor, q_to_seq: torch.Tensor,
                      q_lens: torch.Tensor, num_seqs: int, max_seq_len: int, scale: float,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """Query i (q [n_q, Hq, 256]) attends over the first q_lens[i] tokens of
    sequence q_to_seq[i] (kvq_decode_attn_multi)."""
    for name, t in (("q", q), ("q_to_seq", q_to_seq), ("q_lens", q_lens)):
        _cuda_contig(name, t)
    if q_to_seq.dtype != torch.int32 or q_lens.dtype != torch.int32:
        raise TypeError("q_to_seq and q_lens must be int32")
    n_q, hq, dim = q.shape
    if out is None:
        out = torch.empty((n_q, hq, dim), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_attn_workspace(cache, n_q, hq, max_seq_len)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    d = cache.desc()
    _check("kvq_decode_attn_multi",
           lib().kvq_decode_attn_multi(C.byref(d), _ptr(q), _dtype_code(q), n_q, hq,
                                       _ptr(q_to_seq), _ptr(q_lens), int(num_seqs),
                                       int(max_seq_len), float(scale), _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
    return out


def decode_step(cache: Q4Cache, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                pos: torch.Tensor, max_seq_len: int, scale: float,
                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """Append one token per sequence (k_new, v_new [batch, Hkv, 256] at pos[b])
    and decode over pos[b] + 1 tokens in one call (kvq_decode_step)."""
    for name, t in (("k_new", k_new), ("v_new", v_new), ("q", q), ("pos", pos)):
        _cuda_contig(name, t)
    if pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    if not (k_new.dtype == v_new.dtype == q.dtype):
        raise TypeError("k_new, v_new and q must share one dtype")
    batch, hq, dim = q.shape
    if out is None:
        out = torch.empty((batch, hq, dim), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_attn_workspace(cache, batch, hq, max_seq_len)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    d = cache.desc()
    _check("kvq_decode_step",
           lib().kvq_decode_step(C.byref(d), _ptr(k_new), _ptr(v_new), _ptr(q), _dtype_code(q),
                                 batch, hq, _ptr(pos), int(max_seq_len), float(scale),
                                 _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def decode_attn_noalloc(cache: Q4Cache, q: torch.Tensor, seq_lens: torch.Tensor,
                        max_seq_len: int, scale: float, out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """decode_attn with the split-K scratch taken from the library's fixed
    device array instead of a caller workspace (kvq_decode_attn_noalloc)."""
    _cuda_contig("q", q)
    _cuda_contig("seq_lens", seq_lens)
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    batch, hq, dim = q.shape
    if out is None:
        out = torch.empty((batch, hq, dim), dtype=torch.float32, device=q.device)
    d = cache.desc()
    _check("kvq_decode_attn_noalloc",
           lib().kvq_decode_attn_noalloc(C.byref(d), _ptr(q), _dtype_code(q), batch, hq,
                                         _ptr(seq_lens), int(max_seq_len), float(scale),
                                         _ptr(out), _stream(stream)))
    return out


# --------------------------------------------------------------------------
# Octave
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class OctaveFormat:
    head_size: int
    rope_dim: int
    v_bits: int
    compact: bool = False

    CACHE_DTYPES = {"octave_k3v4": (4, False), "octave_k3v3": (3, False),
                    "octave_k3v3_compact": (3, True)}

    @classmethod
    def from_cache_dtype(cls, cache_dtype: str, head_size: int, rope_dim: int):
        v_bits, compact = cls.CACHE_DTYPES[cache_dtype]
        return cls(head_size, rope_dim, v_bits, compact)

    def desc(self) -> OctaveFmtDesc:
        return OctaveFmtDesc(self.head_size, self.rope_dim, self.v_bits, int(self.compact))

    def layout(self) -> dict:
        out = OctaveLayoutDesc()
        f = self.desc()
        _check("kvq_octave_layout_of", lib().kvq_octave_layout_of(C.byref(f), C.byref(out)))
        return {n: getattr(out, n) for n, _ in OctaveLayoutDesc._fields_}


@functools.lru_cache(maxsize=None)
def _slot_bytes(fmt: OctaveFormat) -> int:
    return fmt.layout()["slot_bytes"]


def _octave_cache_shape(fmt: OctaveFormat, cache: torch.Tensor):
    """(num_blocks, kv heads, block_size) of a cache [num_blocks, Hkv,
    block_size, slot bytes of fmt]; the C ABI takes the slot width from the
    format, so a cache of another width is refused here."""
    if cache.dim() != 4 or cache.shape[3] != _slot_bytes(fmt):
        raise ValueError(f"cache must be [num_blocks, kv heads, block_size, {_slot_bytes(fmt)}] "
                         f"for this format, got {tuple(cache.shape)}")
    return cache.shape[0], cache.shape[1], cache.shape[2]


def octave_codebook(bits: int):
    lut = np.zeros(1 << bits, np.int8)
    mult = C.c_float(0)
    _check("kvq_octave_codebook",
           lib().kvq_octave_codebook(bits, lut.ctypes.data_as(C.c_void_p), C.byref(mult)))
    return lut, float(np.float32(mult.value))


def sign_words(signs) -> np.ndarray:
    """+-1 pattern -> int32 words with bit i set where the sign is -1."""
    neg = (np.asarray(signs) < 0).astype(np.uint64).reshape(-1, 32)
    words = (neg << np.arange(32, dtype=np.uint64)).sum(axis=1).astype(np.uint32)
    return words.view(np.int32).copy()


def octave_quantize(fmt: OctaveFormat, key: torch.Tensor, value: torch.Tensor,
                    slot_mapping: torch.Tensor, cache: torch.Tensor, sign_bits: np.ndarray,
                    stream=None) -> None:
    """key/value [T, Hkv, D] -> slots of cache [num_blocks, Hkv, block_size, slot]."""
    num_blocks, _, block_size = _octave_cache_shape(fmt, cache)
    for n, t in (("key", key), ("value", value), ("slot_mapping", slot_mapping),
                 ("cache", cache)):
        _cuda_contig(n, t)
    if slot_mapping.dtype != torch.int64 or cache.dtype != torch.uint8:
        raise TypeError("slot_mapping must be int64 and cache uint8")
    T, hkv, _ = key.shape
    f = fmt.desc()
    sb = np.ascontiguousarray(sign_bits, dtype=np.int32)
    _check("kvq_octave_quantize",
           lib().kvq_octave_quantize(C.byref(f), _ptr(key), _ptr(value), _dtype_code(key), T, hkv,
                                     _ptr(slot_mapping), _ptr(cache), block_size, num_blocks,
                                     sb.ctypes.data_as(C.c_void_p), _stream(stream)))


def octave_decode_attn_workspace(fmt: OctaveFormat, num_q: int, num_q_heads: int,
                                 max_klen: int) -> int:
    f = fmt.desc()
    return int(lib().kvq_octave_decode_attn_workspace(C.byref(f), num_q, num_q_heads, max_klen))


def octave_decode_attn(fmt: OctaveFormat, query: torch.Tensor, cache: torch.Tensor,
                       block_table: torch.Tensor, q_to_req: torch.Tensor,
                       q_to_klen: torch.Tensor, max_klen: int, scale: float,
                       sign_bits: np.ndarray, out: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    num_blocks, hkv, block_size = _octave_cache_shape(fmt, cache)
    for n, t in (("query", query), ("cache", cache), ("block_table", block_table),
                 ("q_to_req", q_to_req), ("q_to_klen", q_to_klen)):
        _cuda_contig(n, t)
    nq, hq, d = query.shape
    if out is None:
        out = torch.empty((nq, hq, d), dtype=torch.float32, device=query.device)
    if workspace is None:
        nbytes = octave_decode_attn_workspace(fmt, nq, hq, max_klen)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=query.device)
    f = fmt.desc()
    sb = np.ascontiguousarray(sign_bits, dtype=np.int32)
    _check("kvq_octave_decode_attn",
           lib().kvq_octave_decode_attn(
               C.byref(f), _ptr(query), _dtype_code(query), nq, hq, _ptr(cache), hkv, block_size,
               num_blocks, _ptr(block_table), block_table.shape[0], block_table.shape[1],
               _ptr(q_to_req), _ptr(q_to_klen), int(max_klen), float(scale),
               sb.ctypes.data_as(C.c_void_p), _ptr(out), _ptr(workspace),
               workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


# --------------------------------------------------------------------------
# Diagnostics
# --------------------------------------------------------------------------
def device_errors() -> int:
    """Flags recorded on the current device since the last call (cleared by
    reading; synchronizes the device): KVQ_DEVERR_WAIT_TIMEOUT, KVQ_DEVERR_BOUNDS."""
    f = C.c_uint32(0)
    _check("kvq_device_errors", lib().kvq_device_errors(C.byref(f)))
    return int(f.value)


def set_wait_limit(polls: int = -1) -> None:
    """Poll limit of the decode kernels' bounded waits (-1: the default)."""
    _check("kvq_set_wait_limit", lib().kvq_set_wait_limit(int(polls)))

