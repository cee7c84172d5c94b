"""GPU parity of decode under the balanced stream schedule (batches with at
least a quarter-wave of (row, head group) units: every CTA takes an equal run
of all units' tiles and may cross unit boundaries).  Mixed lengths with empty
and one-token rows, fewer tiles than CTAs, all rows empty, paged caches, the
fused step (whose appending CTA is given fewer tiles) and multi-token decode,
over Q4_0 and Q8_0 caches, against the fp64 oracle."""
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


def mixed_lengths(seed, B, T):
    lens = np.random.default_rng(seed).integers(0, T + 1, B).astype(np.int32)
    edge = [0, 1, 63, 64, 65, 127, 128, 129, T]
    lens[:len(edge)] = edge
    return lens


def contiguous(seed, B, H, T, bits):
    k, v = synth.kv_tokens(seed, B, T, H, 256, 0.01, 16.0)
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.contiguous(B, H, T, bits=bits)
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T, bits=bits)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    oc.append(k, v, np.zeros(B, np.int32))
    return gc, oc, k, v


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("G", [4, 8, 16])
def test_stream_contiguous_mixed_lengths(bits, G):
    B, H, T = 40, 2, 600  # 40 rows x >= 2 head groups: stream schedule
    gc, oc, _, _ = contiguous(700 + G + bits, B, H, T, bits)
    lens = mixed_lengths(701, B, T)
    q = synth.to_bf16_bits(synth.queries(702 + G, B, H * G, 256))
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    want = oc.decode_attn(q, lens, 1 / 16)
    assert np.abs(got - want).max() <= ATOL
    assert not np.any(got[lens == 0])


@pytest.mark.parametrize("bits", [4, 8])
def test_stream_fewer_tiles_than_ctas_and_all_empty(bits):
    B, H, G, T = 40, 2, 8, 64
    gc, oc, _, _ = contiguous(710 + bits, B, H, T, bits)
    q = synth.to_bf16_bits(synth.queries(711, B, H * G, 256))
    lens = np.ones(B, np.int32)  # 80 units of one tile: fewer tiles than SMs
    lens[::3] = 5
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    assert np.abs(got - oc.decode_attn(q, lens, 1 / 16)).max() <= ATOL
    zero = np.zeros(B, np.int32)
    got0 = kvq.decode_attn(gc, to_dev(q), to_dev(zero), T, 1 / 16).cpu().numpy()
    assert not np.any(got0)


@pytest.mark.parametrize("bits", [4, 8])
def test_stream_paged_equals_contiguous_and_oracle(bits):
    B, H, G, ps = 40, 2, 8, 64
    lens = mixed_lengths(720, B, 700)
    T = int(lens.max())
    npp = np.array([max((int(L) + ps - 1) // ps, 1) for L in lens])
    bt, n_pages = synth.page_table(721, B, npp, int(npp.max()) + 1, extra_pages=3)
    k, v = synth.kv_tokens(722, B, T, H, 256, 0.01, 16.0)
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    q = synth.to_bf16_bits(synth.queries(723, B, H * G, 256))
    pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), bits=bits)
    cc = kvq.Q4Cache.contiguous(B, H, T, bits=bits)
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps, bits=bits)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        sp = np.zeros(1, np.int32)
        kvq.quantize_append(pc.with_block_table(torch.from_numpy(bt[b:b + 1])),
                            to_dev(k[b:b + 1, :L]), to_dev(v[b:b + 1, :L]), to_dev(sp))
        oc.with_block_table(bt[b:b + 1]).append(k[b:b + 1, :L], v[b:b + 1, :L], sp)
    kvq.quantize_append(cc, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    gp = kvq.decode_attn(pc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    gcn = kvq.decode_attn(cc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    assert np.abs(gp - oc.decode_attn(q, lens, 1 / 16)).max() <= ATOL
    np.testing.assert_array_equal(gp, gcn)  # same tiles, same schedule -> same bits


@pytest.mark.parametrize("bits", [4, 8])
def test_stream_fused_step(bits):
    """40 sequences: the fused step writes the same cache bytes as append, and
    its attention (whose schedule counts the append as extra work) matches the
    oracle and the unfused calls to rounding."""
    B, H, G, T = 40, 2, 8, 640
    gc, oc, _, _ = contiguous(730 + bits, B, H, T, bits)
    pos = np.random.default_rng(731).integers(0, T, B).astype(np.int32)
    pos[:4] = [0, 63, 64, T - 1]
    pos[4] = -1  # no token: zero row
    nk, nv = synth.kv_tokens(732, B, 1, H, 256, 0.01, 16.0)
    nk = np.ascontiguousarray(synth.to_bf16_bits(nk)[:, 0])
    nv = np.ascontiguousarray(synth.to_bf16_bits(nv)[:, 0])
    q = synth.to_bf16_bits(synth.queries(733, B, H * G, 256))
    a = kvq.Q4Cache.contiguous(B, H, T, bits=bits)
    f = kvq.Q4Cache.contiguous(B, H, T, bits=bits)
    for name in PLANES:
        getattr(a, name).copy_(getattr(gc, name))
        getattr(f, name).copy_(getattr(gc, name))
    kvq.quantize_append(a, to_dev(nk[:, None]), to_dev(nv[:, None]), to_dev(pos))
    want_gpu = kvq.decode_attn(a, to_dev(q), to_dev(pos + 1), T, 1 / 16)
    got = kvq.decode_step(f, to_dev(nk), to_dev(nv), to_dev(q), to_dev(pos), T, 1 / 16)
    torch.cuda.synchronize()
    for name in PLANES:
        assert torch.equal(getattr(f, name), getattr(a, name)), name
    # the two schedules group the tokens differently, so the fp32 partial sums
    # (and the Q4_0 zero-point bias removal) round differently
    assert (got - want_gpu).abs().max().item() <= 2e-4
    assert torch.count_nonzero(got[4]) == 0
    # the oracle rejects a negative position; the row attends nothing anyway
    oc.append(nk[:, None], nv[:, None], np.maximum(pos, 0))
    assert np.abs(got.cpu().numpy() - oc.decode_attn(q, pos + 1, 1 / 16)).max() <= ATOL


@pytest.mark.parametrize("bits", [4, 8])
def test_stream_multi_token(bits):
    """48 queries over 6 sequences, each over its own prefix, one query with no
    sequence."""
    B, H, G, T = 6, 2, 4, 900
    gc, oc, _, _ = contiguous(740 + bits, B, H, T, bits)
    rng = np.random.default_rng(741)
    q_to_seq = rng.integers(0, B, 48).astype(np.int32)
    q_to_seq[7] = 99
    q_lens = rng.integers(1, T + 1, 48).astype(np.int32)
    q = synth.to_bf16_bits(synth.queries(742, 48, H * G, 256))
    got = kvq.decode_attn_multi(gc, to_dev(q), to_dev(q_to_seq), to_dev(q_lens), B, T,
                                1 / 16).cpu().numpy()
    for i in range(48):
        s = int(q_to_seq[i])
        if s >= B:
            assert not np.any(got[i])
            continue
        qb = np.zeros((B,) + q.shape[1:], q.dtype)
        qb[s] = q[i]
        lens = np.zeros(B, np.int32)
        lens[s] = q_lens[i]
        assert np.abs(got[i] - oc.decode_attn(qb, lens, 1 / 16)[s]).max() <= ATOL


@pytest.mark.parametrize("bits", [4, 8])
def test_chunked_fallback_many_rows(bits):
    """More than 4096 (row, head group) units: fixed 2048-token chunks handed
    out by the block scheduler."""
    B, H, G, T = 4100, 1, 4, 256
    lens = np.random.default_rng(750).integers(0, T + 1, B).astype(np.int32)
    lens[:4] = [0, 1, 128, T]
    gc, oc, _, _ = contiguous(751 + bits, B, H, T, bits)
    q = synth.to_bf16_bits(synth.queries(752, B, H * G, 256))
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    want = oc.decode_attn(q, lens, 1 / 16)
    assert np.abs(got - want).max() <= ATOL
    assert not np.any(got[lens == 0])
