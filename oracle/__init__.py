"""CPU oracle for the Hadamard-rotated low-bit KV cache -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product path (the CUDA library and
its binding) never does; it fails loudly when its own extension is missing.

The arithmetic lives in ``kvq_oracle.c`` (plain single-threaded C, fp32 where
the pages fix it, fp64 for attention).  This module only compiles it with gcc
and marshals numpy arrays.  Page citations are in the C source:
Strata PR #21 "Q4_0 KV cache + FWHT-256" and the vLLM API page
"vllm.v1.attention.ops.rocm_octave".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_HDR = os.path.join(_HERE, "kvq_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fused multiply-add, IEEE fp32)."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class OctaveFmt(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "head_size", "rope_dim", "v_bits", "compact", "k_rotation_block", "k_wide_dim",
        "nope_dim", "num_k_blocks", "num_rope_blocks", "off_k_nope", "off_v",
        "off_scales", "num_k_scales", "num_scales", "slot_bytes", "kernel_code")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.orc_f32_to_f16.restype = C.c_uint16
        _lib.orc_f32_to_f16.argtypes = [C.c_float]
        _lib.orc_f16_to_f32.restype = C.c_float
        _lib.orc_f16_to_f32.argtypes = [C.c_uint16]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(r, what):
    if r != 0:
        raise ValueError(f"oracle {what} failed with status {r}")


def _dtype_code(a):
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:  # raw bf16 bit patterns
        return 1
    raise TypeError("oracle inputs are float32 or bf16 bit patterns (uint16)")


# ---------------------------------------------------------------- conversions
def f32_to_f16_bits(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_f16_array(_p(x), _p(out), C.c_int64(x.size))
    return out


def f16_bits_to_f32(h):
    h = np.ascontiguousarray(h, dtype=np.uint16).ravel()
    return np.array([lib().orc_f16_to_f32(int(v)) for v in h], np.float32)


# ---------------------------------------------------------------- rotation
def fwht_f32(x, block=256):
    """Orthonormal FWHT over consecutive blocks of the last dim, fp32, page order."""
    y = np.array(x, dtype=np.float32, copy=True, order="C")
    dim = y.shape[-1]
    _check(lib().orc_fwht_f32(_p(y), C.c_int64(y.size // dim), dim, block), "fwht_f32")
    return y


def fwht_f64(x, block=256):
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    dim = y.shape[-1]
    _check(lib().orc_fwht_f64(_p(y), C.c_int64(y.size // dim), dim, block), "fwht_f64")
    return y


# ---------------------------------------------------------------- Q4_0
def q4_0_block(z):
    z = np.ascontiguousarray(z, dtype=np.float32)
    assert z.shape == (32,)
    qs = np.zeros(16, np.uint8)
    d = C.c_uint16(0)
    _check(lib().orc_q4_0_block(_p(z), _p(qs), C.byref(d)), "q4_0_block")
    return qs, int(d.value)


def q4_0_dequant_block(qs, d_bits):
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    out = np.zeros(32, np.float64)
    _check(lib().orc_q4_0_dequant_block(_p(qs), C.c_uint16(d_bits), _p(out)), "dequant")
    return out


def q4_quantize_vectors(x):
    """x: (..., 256) float32 or bf16 bits -> codes (..., 128) u8, scales (..., 8) u16."""
    x = np.ascontiguousarray(x)
    n = x.size // 256
    codes = np.zeros(x.shape[:-1] + (128,), np.uint8)
    scales = np.zeros(x.shape[:-1] + (8,), np.uint16)
    _check(lib().orc_q4_quantize_vectors(_p(x), _dtype_code(x), C.c_int64(n), _p(codes),
                                         _p(scales)), "q4_quantize_vectors")
    return codes, scales


# ---------------------------------------------------------------- Q8_0
def q8_0_block(z):
    z = np.ascontiguousarray(z, dtype=np.float32)
    assert z.shape == (32,)
    qs = np.zeros(32, np.int8)
    d = C.c_uint16(0)
    _check(lib().orc_q8_0_block(_p(z), _p(qs), C.byref(d)), "q8_0_block")
    return qs, int(d.value)


def q8_0_dequant_block(qs, d_bits):
    qs = np.ascontiguousarray(qs, dtype=np.int8)
    out = np.zeros(32, np.float64)
    _check(lib().orc_q8_0_dequant_block(_p(qs), C.c_uint16(d_bits), _p(out)), "q8 dequant")
    return out


def q8_quantize_vectors(x):
    """x: (..., 256) float32 or bf16 bits -> codes (..., 256) int8, scales (..., 8) u16."""
    x = np.ascontiguousarray(x)
    n = x.size // 256
    codes = np.zeros(x.shape[:-1] + (256,), np.int8)
    scales = np.zeros(x.shape[:-1] + (8,), np.uint16)
    _check(lib().orc_q8_quantize_vectors(_p(x), _dtype_code(x), C.c_int64(n), _p(codes),
                                         _p(scales)), "q8_quantize_vectors")
    return codes, scales


# ---------------------------------------------------------------- threads
# The oracle itself is single-threaded C.  For large workloads the calls below
# can split the work into independent units -- (sequence, kv head) for decode,
# (sequence, token range) for append, query tokens for Octave attention, token
# ranges for Octave quantize -- and run the unchanged C function on each unit
# from a pool of host threads (ctypes releases the GIL during the call).  Each
# unit performs exactly the operations, in the same order, that the whole call
# performs for it, so the results are bit-identical to the single call.
def host_threads() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_units(fn, units, threads):
    """fn(unit) for each unit on up to `threads` host threads, results in order."""
    if threads <= 1 or len(units) <= 1:
        return [fn(u) for u in units]
    # fill the oracle's lazily computed codebook cache before any thread runs
    octave_codebook(3)
    octave_codebook(4)
    with ThreadPoolExecutor(min(threads, len(units))) as ex:
        return list(ex.map(fn, units))


class Q4Cache:
    """Oracle-side Q4_0 cache with the documented structure-of-arrays layout
    (bits = 8: the Q8_0 cache, 256 int8 code bytes per row)."""

    def __init__(self, n_rows, n_kv_heads, max_tokens=0, block_table=None, page_size=0,
                 bits=4):
        self.n_kv_heads = n_kv_heads
        self.max_tokens = max_tokens
        self.block_table = (None if block_table is None else
                            np.ascontiguousarray(block_table, dtype=np.int32))
        self.page_size = page_size
        self.max_pages = 0 if block_table is None else self.block_table.shape[1]
        self.bits = bits
        cdt, cw = (np.int8, 256) if bits == 8 else (np.uint8, 128)
        self.k_codes = np.zeros((n_rows, cw), cdt)
        self.v_codes = np.zeros((n_rows, cw), cdt)
        self.k_scales = np.zeros((n_rows, 8), np.uint16)
        self.v_scales = np.zeros((n_rows, 8), np.uint16)

    def with_block_table(self, block_table):
        view = Q4Cache.__new__(Q4Cache)
        view.__dict__.update(self.__dict__)
        view.block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        view.max_pages = view.block_table.shape[1]
        return view

    def _args(self):
        return (_p(self.k_codes), _p(self.k_scales), _p(self.v_codes), _p(self.v_scales),
                self.n_kv_heads, self.max_tokens, _p(self.block_table), self.page_size,
                self.max_pages)

    def _seq_view_args(self, b):
        """Arguments that make sequence b of this cache sequence 0 of a cache
        (same rows, same kv heads)."""
        if self.block_table is None:
            row0 = b * self.n_kv_heads * self.max_tokens
            bt, ps, mp, mt = None, 0, 0, self.max_tokens
            keep = None
        else:
            row0 = 0
            keep = np.ascontiguousarray(self.block_table[b:b + 1])
            bt, ps, mp, mt = keep, self.page_size, self.max_pages, 0
        planes = [a[row0:] for a in (self.k_codes, self.k_scales, self.v_codes, self.v_scales)]
        args = (*[_p(a) for a in planes], self.n_kv_heads, mt, _p(bt), ps, mp)
        return args, (planes, keep)

    def _unit_view_args(self, b, g):
        """Arguments that make (sequence b, kv head g) the only sequence and kv
        head of a paged cache over the same rows: a one-entry block table
        holding page 0 of a view whose base is the unit's first row
        (contiguous), or the sequence's pages times the kv head count with the
        base moved by g pages' worth of rows (paged)."""
        if self.block_table is None:
            row0 = (b * self.n_kv_heads + g) * self.max_tokens
            bt = np.zeros((1, 1), np.int32)
            ps, mp = self.max_tokens, 1
        else:
            row0 = g * self.page_size
            pages = self.block_table[b:b + 1].astype(np.int64)
            bt = np.where(pages < 0, -1, pages * self.n_kv_heads).astype(np.int32)
            ps, mp = self.page_size, self.max_pages
        planes = [a[row0:] for a in (self.k_codes, self.k_scales, self.v_codes, self.v_scales)]
        args = (*[_p(a) for a in planes], 1, 0, _p(bt), ps, mp)
        return args, (planes, bt)

    def append(self, k, v, start_pos, threads=1, chunk=512):
        """Quantize k, v ([batch, t_new, Hkv, 256]) into the cache; with
        threads > 1, (sequence, chunk of tokens) units run in parallel."""
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        assert k.shape == v.shape and k.dtype == v.dtype
        batch, t_new, hkv, d = k.shape
        assert hkv == self.n_kv_heads and d == 256
        sp = np.ascontiguousarray(start_pos, dtype=np.int32)
        fn = lib().orc_q8_append if self.bits == 8 else lib().orc_q4_append
        if threads <= 1:
            _check(fn(*self._args(), _p(k), _p(v), _dtype_code(k), batch, t_new, _p(sp)),
                   "append")
            return

        def unit(u):
            b, i0 = u
            args, keep = self._seq_view_args(b)
            ku = np.ascontiguousarray(k[b:b + 1, i0:i0 + chunk])
            vu = np.ascontiguousarray(v[b:b + 1, i0:i0 + chunk])
            spu = np.array([sp[b] + i0], np.int32)
            return fn(*args, _p(ku), _p(vu), _dtype_code(ku), 1, ku.shape[1], _p(spu))

        units = [(b, i0) for b in range(batch) for i0 in range(0, t_new, chunk)]
        for r in run_units(unit, units, threads):
            _check(r, "append")

    def decode_attn(self, q, seq_lens, scale, threads=1):
        """fp64 decode attention; with threads > 1, (sequence, kv head) units
        run in parallel."""
        q = np.ascontiguousarray(q)
        batch, hq, d = q.shape
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        out = np.zeros((batch, hq, d), np.float64)
        fn = lib().orc_q8_decode_attn if self.bits == 8 else lib().orc_q4_decode_attn
        if threads <= 1:
            _check(fn(*self._args(), _p(q), _dtype_code(q), batch, hq, _p(sl),
                      C.c_double(scale), _p(out)), "decode_attn")
            return out
        G = hq // self.n_kv_heads

        def unit(u):
            b, g = u
            args, keep = self._unit_view_args(b, g)
            qu = np.ascontiguousarray(q[b:b + 1, g * G:(g + 1) * G])
            ou = np.zeros((1, G, d), np.float64)
            r = fn(*args, _p(qu), _dtype_code(qu), 1, G, _p(sl[b:b + 1].copy()),
                   C.c_double(scale), _p(ou))
            return r, ou

        units = [(b, g) for b in range(batch) for g in range(self.n_kv_heads)]
        for (b, g), (r, ou) in zip(units, run_units(unit, units, threads)):
            _check(r, "decode_attn")
            out[b, g * G:(g + 1) * G] = ou[0]
        return out


# ---------------------------------------------------------------- Octave
def lloyd_max(bits):
    c = np.zeros(1 << bits, np.float64)
    b = np.zeros((1 << bits) - 1, np.float64)
    _check(lib().orc_lloyd_max(bits, _p(c), _p(b)), "lloyd_max")
    return c, b


def octave_codebook(bits):
    lut = np.zeros(1 << bits, np.int8)
    mult = C.c_float(0)
    _check(lib().orc_octave_codebook(bits, _p(lut), C.byref(mult)), "octave_codebook")
    return lut, float(np.float32(mult.value))


def octave_format(head_size, rope_dim, v_bits, compact=False):
    f = OctaveFmt()
    _check(lib().orc_octave_format(head_size, rope_dim, v_bits, int(compact), C.byref(f)),
           "octave_format")
    return f.as_dict()


def octave_pack(codes, bits):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(codes.size * bits // 8, np.uint8)
    _check(lib().orc_octave_pack(_p(codes), codes.size, bits, _p(out)), "pack")
    return out


def octave_unpack(packed, n, bits):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros(n, np.uint8)
    _check(lib().orc_octave_unpack(_p(packed), n, bits, _p(out)), "unpack")
    return out


def octave_quantize_lut(x, bits):
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, np.uint8)
    s = C.c_float(0)
    _check(lib().orc_octave_quantize_lut(_p(x), x.size, bits, _p(codes), C.byref(s)), "qlut")
    return codes, float(np.float32(s.value))


def octave_rotate(x, signs, block):
    y = np.array(x, dtype=np.float32, copy=True)
    s = np.ascontiguousarray(signs, dtype=np.float32)
    _check(lib().orc_octave_rotate(_p(y), _p(s), y.size, block), "rotate")
    return y


def octave_unrotate(y, signs, block):
    z = np.array(y, dtype=np.float64, copy=True)
    s = np.ascontiguousarray(signs, dtype=np.float32)
    _check(lib().orc_octave_unrotate_f64(_p(z), _p(s), z.size, block), "unrotate")
    return z


def octave_quantize(key, value, fmt, signs, threads=1, chunk=1024):
    """fmt: (head_size, rope_dim, v_bits, compact). key/value: (T, H, D).
    With threads > 1, chunks of tokens run in parallel."""
    key = np.ascontiguousarray(key)
    value = np.ascontiguousarray(value)
    T, H, D = key.shape
    info = octave_format(*fmt)
    out = np.zeros((T, H, info["slot_bytes"]), np.uint8)
    s = np.ascontiguousarray(signs, dtype=np.float32)

    def unit(t0):
        t1 = min(T, t0 + chunk)
        return lib().orc_octave_quantize(*fmt, _p(key[t0:t1]), _p(value[t0:t1]),
                                         _dtype_code(key), t1 - t0, H, _p(s), _p(out[t0:t1]))

    if threads <= 1:
        _check(lib().orc_octave_quantize(*fmt, _p(key), _p(value), _dtype_code(key), T, H, _p(s),
                                         _p(out)), "octave_quantize")
        return out
    for r in run_units(unit, list(range(0, T, chunk)), threads):
        _check(r, "octave_quantize")
    return out


def octave_dequantize(slots, fmt, signs, rotated=False):
    slots = np.ascontiguousarray(slots, dtype=np.uint8)
    T, H, _ = slots.shape
    D = fmt[0]
    k = np.zeros((T, H, D), np.float64)
    v = np.zeros((T, H, D), np.float64)
    s = np.ascontiguousarray(signs, dtype=np.float32)
    _check(lib().orc_octave_dequantize(*fmt, _p(slots), T, H, _p(s), int(rotated), _p(k),
                                       _p(v)), "octave_dequantize")
    return k, v


def octave_attention(query, cache, block_table, q_to_req, q_to_klen, fmt, scale, signs,
                     threads=1):
    """reference_attention in fp64; with threads > 1, query tokens run in
    parallel."""
    query = np.ascontiguousarray(query)
    cache = np.ascontiguousarray(cache, dtype=np.uint8)
    nq, hq, d = query.shape
    _, hkv, bs, _ = cache.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    qr = np.ascontiguousarray(q_to_req, dtype=np.int32)
    ql = np.ascontiguousarray(q_to_klen, dtype=np.int32)
    s = np.ascontiguousarray(signs, dtype=np.float32)
    out = np.zeros((nq, hq, d), np.float64)

    def unit(i):
        return lib().orc_octave_attention(*fmt, _p(query[i:i + 1]), _dtype_code(query), 1, hq,
                                          _p(cache), C.c_int64(cache.shape[0]), hkv, bs, _p(bt),
                                          bt.shape[1], _p(qr[i:i + 1]), _p(ql[i:i + 1]),
                                          C.c_double(scale), _p(s), _p(out[i:i + 1]))

    if threads <= 1:
        _check(lib().orc_octave_attention(*fmt, _p(query), _dtype_code(query), nq, hq, _p(cache),
                                          C.c_int64(cache.shape[0]), hkv, bs, _p(bt), bt.shape[1],
                                          _p(qr), _p(ql), C.c_double(scale), _p(s), _p(out)),
               "octave_attention")
        return out
    for r in run_units(unit, list(range(nq)), threads):
        _check(r, "octave_attention")
    return out
