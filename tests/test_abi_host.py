"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/kvq.h declares, and its host-only calls and argument
validation behave as documented.  No call here reaches a kernel launch."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from hadamard_rotated_bit_fwht_b200 import build, kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return kvq.lib()


def declared_functions():
    hdr = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", hdr))


def test_exports_match_header(L):
    declared = declared_functions()
    assert declared == set(kvq.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", kvq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert declared <= exported
    # nothing else of ours leaks out
    assert {s for s in exported if s.startswith("kvq")} == declared


def test_status_strings_and_version(L):
    assert kvq.status_string(0) == "ok"
    assert "workspace" in kvq.status_string(3)
    assert L.kvq_version() >= 100


def test_codebook_matches_oracle(L):
    for bits in (3, 4):
        lut, mult = kvq.octave_codebook(bits)
        olut, omult = oracle.octave_codebook(bits)
        np.testing.assert_array_equal(lut, olut)
        assert mult == omult


@pytest.mark.parametrize("fmt", [(128, 64, 4, 0), (128, 64, 3, 0), (128, 64, 3, 1), (256, 64, 4, 0)])
def test_octave_layout_matches_oracle(L, fmt):
    lay = kvq.OctaveFormat(fmt[0], fmt[1], fmt[2], bool(fmt[3])).layout()
    o = oracle.octave_format(*fmt)
    for k in ("off_k_nope", "off_v", "off_scales", "num_scales", "slot_bytes", "kernel_code"):
        assert lay[k] == o[k]


def test_octave_layout_rejects_invalid(L):
    for fmt in [(128, 64, 5, False), (192, 64, 3, True), (128, 32, 4, False)]:
        with pytest.raises(kvq.KVQError) as e:
            kvq.OctaveFormat(*fmt).layout()
        assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


def test_validation_without_launch(L):
    # wrong dim -> unsupported; null pointers -> invalid; no launch happens
    assert L.kvq_rotate(None, 0, None, 4, 128, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_rotate(None, 0, None, 4, 256, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_rotate(None, 0, None, 0, 256, None) == kvq.KVQ_OK  # empty is a no-op
    assert L.kvq_rotate(None, 7, None, 4, 256, None) == kvq.KVQ_ERR_INVALID_ARG
    d = kvq.CacheDesc()
    assert L.kvq_quantize_append(C.byref(d), None, None, 1, 1, 1, None, None) == kvq.KVQ_ERR_INVALID_ARG
    buf = (C.c_uint8 * 4096)()
    p = C.addressof(buf)
    p16 = (p + 15) // 16 * 16
    d = kvq.CacheDesc(p16, p16, p16, p16, 2, 128, 64, 1, None, 0, 0, 0)
    assert L.kvq_quantize_append(C.byref(d), None, None, 1, 1, 1, None, None) == kvq.KVQ_ERR_UNSUPPORTED
    d.head_dim = 256
    # batch larger than the contiguous capacity
    assert L.kvq_quantize_append(C.byref(d), None, None, 1, 2, 1, None, None) == kvq.KVQ_ERR_INVALID_ARG
    # decode: group size 3 unsupported, heads not a multiple invalid, workspace too small
    assert L.kvq_decode_attn(C.byref(d), p16, 1, 1, 6, p16, 64, C.c_float(0.1), p16, None, 0, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_attn(C.byref(d), p16, 1, 1, 5, p16, 64, C.c_float(0.1), p16, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn(C.byref(d), p16, 1, 1, 8, p16, 64, C.c_float(0.1), p16, None, 0, None) == kvq.KVQ_ERR_WORKSPACE
    need = L.kvq_decode_attn_workspace(C.byref(d), 1, 8, 64)
    assert need > 0
    assert L.kvq_decode_attn(C.byref(d), p16, 1, 1, 8, p16, 64, C.c_float(0.1), p16, p16, need - 1, None) == kvq.KVQ_ERR_WORKSPACE
    # code_bits other than 0, 4 or 8 is rejected
    d.code_bits = 5
    assert L.kvq_quantize_append(C.byref(d), p16, p16, 1, 1, 1, p16, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn(C.byref(d), p16, 1, 1, 8, p16, 64, C.c_float(0.1), p16, p16, need, None) == kvq.KVQ_ERR_INVALID_ARG
    d.code_bits = 8
    assert L.kvq_decode_attn(C.byref(d), p16, 1, 1, 6, p16, 64, C.c_float(0.1), p16, None, 0, None) == kvq.KVQ_ERR_UNSUPPORTED
    # paged cache needs a page size that is a multiple of 64
    d2 = kvq.CacheDesc(p16, p16, p16, p16, 2, 256, 0, 0, p16, 48, 4, 8)
    assert L.kvq_quantize_append(C.byref(d2), p16, p16, 1, 1, 1, p16, None) == kvq.KVQ_ERR_INVALID_ARG
    # octave: head 256 is a valid format this build does not implement
    f = kvq.OctaveFormat(256, 64, 3, True).desc()
    sb = np.zeros(8, np.int32)
    assert L.kvq_octave_quantize(C.byref(f), p16, p16, 1, 1, 1, p16, p16, 16, 1,
                                 sb.ctypes.data_as(C.c_void_p), None) == kvq.KVQ_ERR_UNSUPPORTED


def test_sign_words_marshalling():
    s = np.ones(128, np.float32)
    s[[0, 33, 127]] = -1
    w = kvq.sign_words(s)
    assert w.dtype == np.int32 and w.shape == (4,)
    assert w[0] == 1 and w[1] == 2 and w[3] == np.int32(np.uint32(1 << 31).view(np.int32))


def test_noalloc_checks_arguments_before_its_size(L):
    hdr = open(os.path.join(ROOT, "include", "kvq.h")).read()
    m = re.search(r"#define KVQ_DECODE_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == kvq.KVQ_DECODE_NOALLOC_SCRATCH_BYTES
    buf = (C.c_uint8 * 4096)()
    p16 = (C.addressof(buf) + 15) // 16 * 16
    # 108 sequences x 8 kv heads, 64 q heads (group 8): valid, but its stream-
    # schedule workspace is above the fixed array -> refused before any launch
    d = kvq.CacheDesc(p16, p16, p16, p16, 8, 256, 64, 108, None, 0, 0, 0)
    assert L.kvq_decode_attn_workspace(C.byref(d), 108, 64, 64) > kvq.KVQ_DECODE_NOALLOC_SCRATCH_BYTES

    def call(dtype=1, hq=64, q=p16, batch=108):
        return L.kvq_decode_attn_noalloc(C.byref(d), q, dtype, batch, hq, p16, 64, C.c_float(0.1),
                                         p16, None)

    assert call() == kvq.KVQ_ERR_WORKSPACE
    assert call(dtype=7) == kvq.KVQ_ERR_INVALID_ARG
    assert call(q=None) == kvq.KVQ_ERR_INVALID_ARG
    assert call(hq=8 * 32) == kvq.KVQ_ERR_UNSUPPORTED
    assert call(batch=109) == kvq.KVQ_ERR_INVALID_ARG  # above the contiguous capacity
    assert call(batch=0) == kvq.KVQ_OK


def test_device_error_calls_validate_on_host(L):
    assert L.kvq_device_errors(None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_set_wait_limit(-2) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_set_wait_limit(-1) == kvq.KVQ_OK


def test_octave_bindings_check_the_slot_width_first(L):
    """The C ABI takes the slot width from the format; the bindings refuse a
    cache of another width before any device check or library call."""
    import torch
    F = kvq.OctaveFormat(128, 64, 3)  # 112-byte slots
    cache = torch.zeros((1, 2, 16, 128), dtype=torch.uint8)
    k = torch.zeros((1, 2, 128), dtype=torch.bfloat16)
    i32 = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="cache must be"):
        kvq.octave_quantize(F, k, k, torch.zeros(1, dtype=torch.int64), cache, np.zeros(4))
    with pytest.raises(ValueError, match="cache must be"):
        kvq.octave_decode_attn(F, torch.zeros((1, 4, 128)), cache, i32.view(1, 1), i32, i32, 16,
                               0.1, np.zeros(4))
    with pytest.raises(ValueError, match="cache must be"):  # not 4-D
        kvq.octave_quantize(F, k, k, torch.zeros(1, dtype=torch.int64), cache.view(-1),
                            np.zeros(4))
