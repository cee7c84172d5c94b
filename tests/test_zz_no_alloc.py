"""kvq_decode_attn_noalloc: decode attention for callers that cannot give the
library device scratch memory (a plugin interface that passes only its
tensors, a C host without a device allocator, a decode loop that must not call
cudaMalloc).  Its split-K partials live in a fixed device array inside the
library; this file checks, through the C ABI, that its output is bit-identical
to kvq_decode_attn with a caller workspace on two calls in a row (both calls
run the same plan and the same deterministic kernels), under both work
schedules, and that a valid shape too large for the array is refused before
any launch while a bad argument gets the status kvq_decode_attn gives it.

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


def _dev(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def _noalloc(L, desc, q, lens_d, n_q_heads, max_len, scale):
    B = q.shape[0]
    got = torch.full((B, n_q_heads, 256), float("nan"), device="cuda")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.kvq_decode_attn_noalloc(C.byref(desc), C.c_void_p(q.data_ptr()), kvq.KVQ_BF16, B,
                                   n_q_heads, C.c_void_p(lens_d.data_ptr()), max_len,
                                   C.c_float(scale), C.c_void_p(got.data_ptr()), stream)
    assert st == kvq.KVQ_OK, kvq.status_string(st)
    return got


@pytest.mark.parametrize("B,H,G,T,calls", [
    # 6 (row, head group) units: one wave of equal splits per row
    (3, 2, 8, 3000, ([3000, 1234, 17], [64, 2999, 3000])),
    # 40 units: the balanced stream schedule, ragged lengths including empty rows
    (40, 1, 8, 2500, (None, None)),
])
def test_noalloc_matches_workspace_entry_point(B, H, G, T, calls):
    build.build()
    L = kvq.lib()
    k, v = synth.kv_tokens(707 + B, B, T, H, 256, 0.01, 16.0)
    cache = kvq.Q4Cache.contiguous(B, H, T)
    kvq.quantize_append(cache, _dev(synth.to_bf16_bits(k)), _dev(synth.to_bf16_bits(v)),
                        torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = _dev(synth.to_bf16_bits(synth.queries(708 + B, B, H * G, 256)))
    desc = cache.desc()
    rng = np.random.default_rng(B)
    for call, lens in enumerate(calls):
        if lens is None:
            lens = rng.integers(0, T + 1, size=B)
            lens[rng.integers(0, B)] = 0
            lens[rng.integers(0, B)] = T
        lens_d = torch.tensor(np.asarray(lens), dtype=torch.int32, device="cuda")
        want = kvq.decode_attn(cache, q, lens_d, T, 1 / 16)
        got = _noalloc(L, desc, q, lens_d, H * G, T, 1 / 16)
        torch.cuda.synchronize()
        assert torch.equal(got, want), (
            f"call {call}: max abs difference {(got - want).abs().max().item()}")


def test_noalloc_refuses_oversize_shape_and_checks_arguments_first():
    build.build()
    L = kvq.lib()
    # 8 kv heads with 64 query heads (group 8): a supported shape.  108
    # sequences are 864 (row, head group) units under the stream schedule,
    # whose workspace is above the fixed array.
    B, Hkv, Hq, T = 108, 8, 64, 64
    cache = kvq.Q4Cache.contiguous(B, Hkv, T)
    desc = cache.desc()
    need = L.kvq_decode_attn_workspace(C.byref(desc), B, Hq, T)
    assert need > kvq.KVQ_DECODE_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, 256), dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, Hq, 256), dtype=torch.float32, device="cuda")

    def call(dtype=kvq.KVQ_BF16, n_q_heads=Hq, q_ptr=q.data_ptr()):
        return L.kvq_decode_attn_noalloc(C.byref(desc), C.c_void_p(q_ptr), dtype, B, n_q_heads,
                                         C.c_void_p(lens.data_ptr()), T, C.c_float(0.1),
                                         C.c_void_p(out.data_ptr()), None)

    assert call() == kvq.KVQ_ERR_WORKSPACE
    # bad arguments report what kvq_decode_attn reports, not the size
    assert call(dtype=7) == kvq.KVQ_ERR_INVALID_ARG
    assert call(q_ptr=0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(n_q_heads=8 * 32) == kvq.KVQ_ERR_UNSUPPORTED  # group 32
    torch.cuda.synchronize()
    assert not out.any().item(), "a refused call launched nothing"
