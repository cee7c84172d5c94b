"""The device error word (kvq_device_errors) and the bounded waits of the
decode kernels, exercised without a fault: with the poll limit at 0 a wait on
a tile still in flight gives up at once, the kernel records
KVQ_DEVERR_WAIT_TIMEOUT, drains its own copies and returns; the next call with
the default limit is exact again and the word reads clean."""
import numpy as np
import pytest
import torch

from hadamard_rotated_bit_fwht_b200 import build, kvq, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    kvq.lib()
    kvq.set_wait_limit(-1)
    yield
    kvq.set_wait_limit(-1)


def _case(bits):
    B, H, G, T = 1, 4, 8, 65536
    k, v = synth.kv_tokens(515, B, T, H, 256, 0.01, 16.0)
    cache = kvq.Q4Cache.contiguous(B, H, T, bits=bits)
    dev = lambda a: torch.from_numpy(synth.to_bf16_bits(a)).view(torch.bfloat16).cuda()
    kvq.quantize_append(cache, dev(k), dev(v), torch.zeros(B, dtype=torch.int32, device="cuda"))
    q = dev(synth.queries(516, B, H * G, 256))
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    return cache, q, lens, T


@pytest.mark.parametrize("bits", [4, 8])
def test_wait_timeout_is_reported_and_recovers(bits):
    cache, q, lens, T = _case(bits)
    want = kvq.decode_attn(cache, q, lens, T, 1 / 16)
    assert kvq.device_errors() == 0
    kvq.set_wait_limit(0)
    try:
        got = kvq.decode_attn(cache, q, lens, T, 1 / 16)
        flags = kvq.device_errors()
    finally:
        kvq.set_wait_limit(-1)
    assert flags & kvq.KVQ_DEVERR_WAIT_TIMEOUT
    assert torch.isnan(got).any(), "a CTA that gave up leaves NaN partial results"
    again = kvq.decode_attn(cache, q, lens, T, 1 / 16)
    assert kvq.device_errors() == 0
    assert torch.equal(again, want)


def test_octave_wait_timeout_is_reported_and_recovers():
    """The Octave k3v4 decode with 256-token blocks stages its tiles by tensor
    copies behind bounded mbarrier waits: the same timeout path."""
    F = kvq.OctaveFormat(128, 64, 4)
    B, Hkv, Hq, T, bs = 2, 2, 8, 8192, 256
    nblk = B * T // bs
    k = synth.to_bf16_bits(synth.gaussian(517, (B * T, Hkv, 128)))
    v = synth.to_bf16_bits(synth.gaussian(518, (B * T, Hkv, 128)))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    kd, vd = dev(k).view(torch.bfloat16), dev(v).view(torch.bfloat16)
    cache = torch.zeros((nblk, Hkv, bs, 128), dtype=torch.uint8, device="cuda")
    signs = kvq.sign_words(synth.sign_pattern(128))
    kvq.octave_quantize(F, kd, vd, torch.arange(B * T, dtype=torch.int64, device="cuda"), cache,
                        signs)
    bt = torch.arange(nblk, dtype=torch.int32, device="cuda").view(B, T // bs)
    q = dev(synth.queries(519, B, Hq, 128)).to(torch.bfloat16)
    q2r = torch.arange(B, dtype=torch.int32, device="cuda")
    q2l = torch.full((B,), T, dtype=torch.int32, device="cuda")

    def run():
        return kvq.octave_decode_attn(F, q, cache, bt, q2r, q2l, T, 128 ** -0.5, signs)

    want = run()
    assert kvq.device_errors() == 0
    kvq.set_wait_limit(0)
    try:
        got = run()
        flags = kvq.device_errors()
    finally:
        kvq.set_wait_limit(-1)
    assert flags & kvq.KVQ_DEVERR_WAIT_TIMEOUT
    assert torch.isnan(got).any(), "a CTA that gave up leaves NaN partial results"
    again = run()
    assert kvq.device_errors() == 0
    assert torch.equal(again, want)


def test_wait_limit_validation():
    with pytest.raises(kvq.KVQError):
        kvq.set_wait_limit(-2)
