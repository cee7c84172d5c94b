"""GPU parity of the fused decode step (kvq_decode_step): appending one token
per sequence and attending over the sequence including it, in one call, must
leave the cache and produce the output bit-identical to kvq_quantize_append
followed by kvq_decode_attn, and match the oracle like those calls do."""
import numpy as np
import pytest
import torch

import oracle
from hadamard_rotated_bit_fwht_b200 import build, kvq, synth

pytestmark = pytest.mark.gpu
ATOL = 2e-3  # attention tolerance (max-abs vs the fp64 oracle)
PLANES = ("k_codes", "v_codes", "k_scales", "v_scales")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    kvq.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def to_dev(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def copy_planes(dst, src):
    for name in PLANES:
        getattr(dst, name).copy_(getattr(src, name))


def assert_planes_equal(a, b):
    for name in PLANES:
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def inputs(seed, B, H, G, T, dt):
    k, v = synth.kv_tokens(seed, B, T, H, 256, 0.01, 16.0)
    q = synth.queries(seed + 1, B, H * G, 256)
    nk, nv = synth.kv_tokens(seed + 2, B, 1, H, 256, 0.01, 16.0)  # the new tokens
    cvt = synth.to_bf16_bits if dt == "bf16" else (lambda x: x)
    return cvt(k), cvt(v), cvt(q), np.ascontiguousarray(cvt(nk)[:, 0]), np.ascontiguousarray(cvt(nv)[:, 0])


@pytest.mark.parametrize("G", [4, 8, 16])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_step_equals_append_then_decode(G, dt):
    """Contiguous cache: the new token of each sequence overwrites position
    pos[b] (different data from the prefill there) and the sequence is
    attended over pos[b] + 1 tokens."""
    B, H, T = 3, 2, 1500
    pos = np.array([1000, 37, 1499], np.int32)
    k, v, q, new_k, new_v = inputs(300 + G, B, H, G, T, dt)
    base = kvq.Q4Cache.contiguous(B, H, T)
    kvq.quantize_append(base, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T)
    oc.append(k, v, np.zeros(B, np.int32))
    # unfused: append + decode
    a = kvq.Q4Cache.contiguous(B, H, T)
    copy_planes(a, base)
    kvq.quantize_append(a, to_dev(new_k[:, None]), to_dev(new_v[:, None]), to_dev(pos))
    want_gpu = kvq.decode_attn(a, to_dev(q), to_dev(pos + 1), T, 1 / 16)
    # fused
    f = kvq.Q4Cache.contiguous(B, H, T)
    copy_planes(f, base)
    got = kvq.decode_step(f, to_dev(new_k), to_dev(new_v), to_dev(q), to_dev(pos), T, 1 / 16)
    torch.cuda.synchronize()
    assert_planes_equal(f, a)
    assert torch.equal(got, want_gpu)
    oc.append(new_k[:, None], new_v[:, None], pos)
    want = oc.decode_attn(q, pos + 1, 1 / 16)
    assert np.abs(got.cpu().numpy() - want).max() <= ATOL


def test_step_paged_and_out_of_range_positions():
    """Paged cache with a shuffled table and 64-token pages; one position is
    -1 (nothing appended, zero row) and one lies past the pages the table
    maps for it (nothing appended, the length is clamped to the capacity)."""
    B, H, G, ps = 4, 2, 8, 64
    lens = np.array([130, 64, 5, 256], np.int32)
    T = 256
    npp = np.array([(int(L) + 1 + ps - 1) // ps for L in lens])
    npp[3] = (int(lens[3]) + ps - 1) // ps  # sequence 3: no page for the new token
    maxp = int(npp.max()) + 1
    bt, n_pages = synth.page_table(17, B, npp, maxp, extra_pages=2)
    bt[3, npp[3]:] = -1
    k, v, q, new_k, new_v = inputs(400, B, H, G, T, "bf16")
    base = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    for b in range(B):
        L = int(lens[b])
        kvq.quantize_append(base.with_block_table(torch.from_numpy(bt[b:b + 1])),
                            to_dev(k[b:b + 1, :L]), to_dev(v[b:b + 1, :L]),
                            to_dev(np.zeros(1, np.int32)))
    pos = lens.copy()
    pos[1] = -1
    maxlen = int(lens.max()) + 1
    a = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    copy_planes(a, base)
    kvq.quantize_append(a, to_dev(new_k[:, None]), to_dev(new_v[:, None]), to_dev(pos))
    want_gpu = kvq.decode_attn(a, to_dev(q), to_dev(pos + 1), maxlen, 1 / 16)
    f = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    copy_planes(f, base)
    got = kvq.decode_step(f, to_dev(new_k), to_dev(new_v), to_dev(q), to_dev(pos), maxlen, 1 / 16)
    torch.cuda.synchronize()
    assert_planes_equal(f, a)
    assert torch.equal(got, want_gpu)
    assert torch.count_nonzero(got[1]) == 0
    # the oracle over the same paged layout: the new tokens of sequences 0 and
    # 2 appended, none for sequence 1 (position -1, zero row) or sequence 3
    # (no page for its position: its length is clamped to the 256 tokens its
    # pages hold)
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    for b in range(B):
        L = int(lens[b])
        oc.with_block_table(bt[b:b + 1]).append(k[b:b + 1, :L], v[b:b + 1, :L],
                                                np.zeros(1, np.int32))
    for b in (0, 2):
        oc.with_block_table(bt[b:b + 1]).append(new_k[b:b + 1, None], new_v[b:b + 1, None],
                                                pos[b:b + 1])
    for name in PLANES:
        g = getattr(f, name).cpu().numpy()
        assert np.array_equal(g.view(np.uint16) if name.endswith("scales") else g,
                              getattr(oc, name)), name
    olens = np.array([pos[0] + 1, 0, pos[2] + 1, npp[3] * ps], np.int32)
    want = oc.decode_attn(q, olens, 1 / 16)
    assert np.abs(got.cpu().numpy() - want).max() <= ATOL
