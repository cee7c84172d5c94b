"""GPU parity with cache planes larger than 4 GB: the pages (or Octave blocks)
the sequences use sit below and above byte offset 2^32 of their plane, one of
them starting exactly there, so every row and slot address goes through the
64-bit offset arithmetic of the append, the fused append of the decode step,
the TMA tile loads and the cp.async / bulk loads.  The oracle holds the same
tokens in a compact page table; rows are compared page by page."""
import numpy as np
import pytest
import torch

import oracle
from hadamard_rotated_bit_fwht_b200 import build, kvq, synth

pytestmark = pytest.mark.gpu
ATOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    kvq.lib()
    yield
    torch.cuda.empty_cache()


def to_dev(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def _page_rows(pages, H, ps):
    """Row indices of the given physical pages, page by page, head by head."""
    p = np.asarray(pages, np.int64)[:, None, None]
    h = np.arange(H, dtype=np.int64)[None, :, None]
    t = np.arange(ps, dtype=np.int64)[None, None, :]
    return ((p * H + h) * ps + t).reshape(-1)


@pytest.mark.parametrize("bits", [4, 8])
def test_paged_cache_beyond_4gb(bits):
    """Two sequences (1500 and 777 tokens, 8 kv heads, GQA 4, 256-token
    pages) in a paged Q4_0 / Q8_0 cache whose code planes hold 4.7 GB each:
    1499 and 776 tokens appended by kvq_quantize_append, the last token of
    each by kvq_decode_step.  Every row of the used pages bit-exact, all
    outputs within 2e-3 of the oracle."""
    H, Hq, ps = 8, 32, 256
    row_bytes = 128 if bits == 4 else 256
    edge = (1 << 32) // (H * ps * row_bytes)  # the page that starts at byte 2^32
    n_pages = edge + edge // 10
    bt = np.array([[n_pages - 1, 3, edge, n_pages - 2, edge // 2, edge + 7],
                   [n_pages - 3, 0, edge - 1, n_pages - 4, -1, -1]], np.int32)
    lens = np.array([1500, 777], np.int32)
    gc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), bits=bits)
    assert gc.k_codes.numel() > (1 << 32)
    bt_o = np.array([[0, 1, 2, 3, 4, 5], [6, 7, 8, 9, -1, -1]], np.int32)
    oc = oracle.Q4Cache(10 * H * ps, H, block_table=bt_o, page_size=ps, bits=bits)
    k, v = synth.kv_tokens(913, 2, 1500, H, 256, 0.01, 16.0)
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    for b in range(2):
        L = int(lens[b]) - 1
        kvq.quantize_append(gc.with_block_table(torch.from_numpy(bt[b:b + 1])),
                            to_dev(kb[b:b + 1, :L]), to_dev(vb[b:b + 1, :L]),
                            to_dev(np.zeros(1, np.int32)))
        oc.with_block_table(bt_o[b:b + 1]).append(kb[b:b + 1, :L + 1], vb[b:b + 1, :L + 1],
                                                  np.zeros(1, np.int32))
    q = synth.to_bf16_bits(synth.queries(914, 2, Hq, 256))
    last = lens - 1
    got = kvq.decode_step(gc, to_dev(kb[np.arange(2), last]), to_dev(vb[np.arange(2), last]),
                          to_dev(q), to_dev(last.astype(np.int32)), int(lens.max()),
                          1 / 16).cpu().numpy()
    for b in range(2):
        n = (int(lens[b]) + ps - 1) // ps
        rg = torch.from_numpy(_page_rows(bt[b, :n], H, ps)).cuda()
        ro = _page_rows(bt_o[b, :n], H, ps)
        for name in ("k_codes", "v_codes", "k_scales", "v_scales"):
            g = getattr(gc, name).index_select(0, rg).cpu().numpy()
            o = getattr(oc, name)[ro]
            if name.endswith("scales"):
                g = g.view(np.uint16)
            bad = np.nonzero(np.any(g.view(o.dtype) != o, axis=-1))[0]
            assert bad.size == 0, f"sequence {b} {name}: {bad.size} rows differ"
    want = oc.decode_attn(q, lens, 1 / 16)
    err = np.abs(got - want).max()
    assert err <= ATOL, f"max abs error {err}"


@pytest.mark.parametrize("v_bits,bs", [(4, 256), (4, 16), (3, 256)])
def test_octave_cache_beyond_4gb(v_bits, bs):
    """One request of 3000 tokens in an Octave cache of 4.7 GB (8 kv heads;
    block ids below, at and above byte 2^32; 256-token blocks take the TMA
    tiles, 16-token blocks the cp.async rows, k3v3 the SIMT kernel): slots
    bit-exact, the 32 head outputs within 2e-3 of the oracle."""
    fmt = (128, 64, v_bits, 0)
    F = kvq.OctaveFormat(128, 64, v_bits)
    Hkv, Hq, T = 8, 32, 3000
    sbytes = F.layout()["slot_bytes"]  # 128 for k3v4, 112 for k3v3
    blk_bytes = Hkv * bs * sbytes
    edge = -(-(1 << 32) // blk_bytes)  # the first block at or past byte 2^32
    nblk = edge + edge // 10
    n = (T + bs - 1) // bs
    fixed = np.array([nblk - 1, edge, edge - 1, 0], np.int64)
    rest = np.setdiff1d(np.random.default_rng(bs).choice(nblk, 2 * n, replace=False), fixed)
    blocks = np.concatenate([fixed, rest[:n - fixed.size]]).astype(np.int32)
    np.random.default_rng(v_bits).shuffle(blocks)
    bt = blocks[None, :]
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, sbytes), dtype=torch.uint8, device="cuda")
    assert cache.numel() > (1 << 32)
    k, v = synth.kv_tokens(915, 1, T, Hkv, 128, 0.01, 16.0)
    kb, vb = synth.to_bf16_bits(k[0]), synth.to_bf16_bits(v[0])
    slot = (blocks[np.arange(T) // bs].astype(np.int64) * bs + np.arange(T) % bs)
    kvq.octave_quantize(F, to_dev(kb), to_dev(vb), to_dev(slot), cache, kvq.sign_words(signs))
    want_slots = oracle.octave_quantize(kb, vb, fmt, signs)  # (T, Hkv, slot bytes)
    got_slots = cache.index_select(0, torch.from_numpy(blocks).long().cuda()).cpu().numpy()
    got_slots = got_slots.transpose(0, 2, 1, 3).reshape(n * bs, Hkv, sbytes)[:T]
    assert np.array_equal(got_slots, want_slots)
    # the oracle attends over its own slots, in blocks 0..n-1
    oc = np.zeros((n * bs, Hkv, sbytes), np.uint8)
    oc[:T] = want_slots
    oc = oc.reshape(n, bs, Hkv, sbytes).transpose(0, 2, 1, 3).copy()
    q = synth.to_bf16_bits(synth.queries(916, 1, Hq, 128))
    q2r = np.zeros(1, np.int32)
    q2l = np.full(1, T, np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q), cache, to_dev(bt), to_dev(q2r), to_dev(q2l), T,
                                 128 ** -0.5, kvq.sign_words(signs)).cpu().numpy()
    del cache
    want = oracle.octave_attention(q, oc, np.arange(n, dtype=np.int32)[None], q2r, q2l, fmt,
                                   128 ** -0.5, signs)
    err = np.abs(got - want).max()
    assert err <= ATOL, f"max abs error {err}"
