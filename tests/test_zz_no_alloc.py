"""kvq_decode_attn_noalloc: decode attention for callers that cannot give the
library device scratch memory (a plugin interface that passes only its
tensors, a C host without a device allocator, a decode loop that must not call
cudaMalloc).  Its split-K partials live in a fixed device array inside the
library; this file checks, through the C ABI, that its output matches
kvq_decode_attn with a caller workspace on two calls in a row, and that a
shape too large for the array is refused before any launch.

Kept in a file that pytest collects last, so a stop-at-first-failure run has
already run every other test.  It passes alone in a fresh process and after the
other tests: the first call on the device does the one-time address lookup,
and each call overwrites the records it reads.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from hadamard_rotated_bit_fwht_b200 import build, kvq, synth

pytestmark = pytest.mark.gpu
ATOL = 2e-3  # the tolerance of the decode parity tests


def _dev(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def test_noalloc_matches_workspace_entry_point():
    build.build()
    L = kvq.lib()
    B, H, G, T = 3, 2, 8, 3000
    k, v = synth.kv_tokens(707, B, T, H, 256, 0.01, 16.0)
    cache = kvq.Q4Cache.contiguous(B, H, T)
    kvq.quantize_append(cache, _dev(synth.to_bf16_bits(k)), _dev(synth.to_bf16_bits(v)),
                        torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = _dev(synth.to_bf16_bits(synth.queries(708, B, H * G, 256)))
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    desc = cache.desc()
    for call, lens in enumerate(([3000, 1234, 17], [64, 2999, 3000])):
        lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
        want = kvq.decode_attn(cache, q, lens_d, T, 1 / 16)
        got = torch.full((B, H * G, 256), float("nan"), device="cuda")
        st = L.kvq_decode_attn_noalloc(C.byref(desc), C.c_void_p(q.data_ptr()), kvq.KVQ_BF16,
                                       B, H * G, C.c_void_p(lens_d.data_ptr()), T,
                                       C.c_float(1 / 16), C.c_void_p(got.data_ptr()), stream)
        assert st == kvq.KVQ_OK, kvq.status_string(st)
        torch.cuda.synchronize()
        err = (got - want).abs().max().item()
        assert err <= ATOL, f"call {call}: max abs difference {err}"


def test_noalloc_refuses_oversize_shape():
    build.build()
    L = kvq.lib()
    cache = kvq.Q4Cache.contiguous(1, 1, 64)
    desc = cache.desc()
    # 4096 sequences x 64 q heads of 1M tokens need far more than the array
    need = L.kvq_decode_attn_workspace(C.byref(desc), 4096, 64, 1 << 20)
    assert need > kvq.lib().kvq_decode_attn_workspace(C.byref(desc), 1, 8, 64)
    st = L.kvq_decode_attn_noalloc(C.byref(desc), C.c_void_p(1 << 12), kvq.KVQ_BF16, 4096, 64,
                                   C.c_void_p(1 << 12), 1 << 20, C.c_float(0.1),
                                   C.c_void_p(1 << 12), None)
    assert st == kvq.KVQ_ERR_WORKSPACE
