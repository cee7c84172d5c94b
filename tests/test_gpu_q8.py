"""GPU parity of the Q8_0 + FWHT-256 cache (code_bits 8) against the CPU
oracle, through the C ABI: codes and scales bit-identical to the oracle's
Q8_0 of the rotated vectors; attention within 2e-3 max-abs of the oracle's
fp64 evaluation of the same cache; the fused step and multi-token decode
equal to their unfused forms."""
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


def host_plane(gpu, name):
    g = getattr(gpu, name).cpu().numpy()
    return g.view(np.uint16) if name.endswith("scales") else g.view(np.int8)


def compare_cache(gpu, orc, rows=None):
    for name in PLANES:
        g, o = host_plane(gpu, name), getattr(orc, name)
        if rows is not None:
            g, o = g[rows], o[rows]
        bad = np.nonzero(np.any(g != o, axis=-1))[0]
        assert bad.size == 0, f"{name}: {bad.size} rows differ, first {bad[:5]}"


# ------------------------------------------------------------------ append
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_append_tiny_contiguous(dt):
    """Tiny workload shape (1 sequence, 1 kv head, 512 tokens, four x20
    outlier channels), quantized in three appends."""
    W = synth.WORKLOADS["tiny"]
    ch = np.array(W["outlier_channels"])
    k = synth.apply_outliers(synth.gaussian(2010, (1, 512, 1, 256)), ch, W["outlier_factor"])
    v = synth.apply_outliers(synth.gaussian(2020, (1, 512, 1, 256)), ch, W["outlier_factor"])
    if dt == "bf16":
        k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.contiguous(1, 1, 512, bits=8)
    oc = oracle.Q4Cache(512, 1, max_tokens=512, bits=8)
    for lo, hi in [(0, 300), (300, 511), (511, 512)]:
        sp = np.array([lo], np.int32)
        kvq.quantize_append(gc, to_dev(k[:, lo:hi]), to_dev(v[:, lo:hi]), to_dev(sp))
        oc.append(k[:, lo:hi], v[:, lo:hi], sp)
    torch.cuda.synchronize()
    compare_cache(gc, oc)


def test_append_ragged_batch_skip_and_zero_blocks():
    """Different start positions, positions past the capacity skipped, and an
    all-zero vector (scales 0, codes 0)."""
    B, H, T, cap = 3, 5, 37, 64
    k = synth.gaussian(261, (B, T, H, 256)) * np.float32(4)
    k[0, 3, 1, :] = 0.0  # an all-zero vector: all-zero blocks after the rotation
    k = synth.to_bf16_bits(k)
    v = synth.to_bf16_bits(synth.gaussian(262, (B, T, H, 256)))
    sp = np.array([0, 20, 40], np.int32)
    gc = kvq.Q4Cache.contiguous(B, H, cap, bits=8)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(sp))
    torch.cuda.synchronize()
    g = {n: host_plane(gc, n) for n in PLANES}
    for b in range(B):
        n = min(T, cap - int(sp[b]))
        one = oracle.Q4Cache(H * cap, H, max_tokens=cap, bits=8)
        one.append(k[b:b + 1, :n], v[b:b + 1, :n], sp[b:b + 1])
        for h in range(H):
            base_g, base_o = (b * H + h) * cap, h * cap
            for name in PLANES:
                assert np.array_equal(g[name][base_g:base_g + cap],
                                      getattr(one, name)[base_o:base_o + cap]), (b, h, name)
    row = (0 * H + 1) * cap + 3
    assert not np.any(g["k_scales"][row]) and not np.any(g["k_codes"][row])


def paged_setup(seed, B, lens, ps, extra=3):
    npp = [(int(L) + ps - 1) // ps for L in lens]
    return synth.page_table(seed, B, np.array(npp), max(npp) + 1, extra_pages=extra)


def append_paged(gpu, orc, k, v, lens, bt):
    for b in range(len(lens)):
        L = int(lens[b])
        sp = np.zeros(1, np.int32)
        kvq.quantize_append(gpu.with_block_table(torch.from_numpy(bt[b:b + 1])),
                            to_dev(k[b:b + 1, :L]), to_dev(v[b:b + 1, :L]), to_dev(sp))
        if orc is not None:
            orc.with_block_table(bt[b:b + 1]).append(k[b:b + 1, :L], v[b:b + 1, :L], sp)


def test_append_paged_bitexact():
    B, H, ps = 4, 2, 64
    lens = np.array([64, 130, 7, 200], np.int32)
    T = int(lens.max())
    bt, n_pages = paged_setup(209, B, lens, ps)
    k = synth.to_bf16_bits(synth.gaussian(271, (B, T, H, 256)) * 2)
    v = synth.to_bf16_bits(synth.gaussian(272, (B, T, H, 256)))
    gc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), bits=8)
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps, bits=8)
    append_paged(gc, oc, k, v, lens, bt)
    torch.cuda.synchronize()
    compare_cache(gc, oc)


def test_append_stress_bitexact():
    """2^18 vectors per tensor with magnitudes over six decades and an outlier
    channel: every code and scale bit-identical (round-half-away ties and the
    folded 1/16 included)."""
    n = 1 << 18
    x = synth.gaussian(323, (2, n, 256))
    mag = np.exp(np.random.default_rng(15).uniform(np.log(1e-3), np.log(1e3), (2, n, 1))).astype(np.float32)
    x = (x * mag).astype(np.float32)
    x[:, ::17, 200] *= 30
    xb = synth.to_bf16_bits(x)
    gc = kvq.Q4Cache.contiguous(1, 1, n, bits=8)
    kvq.quantize_append(gc, to_dev(xb[0].reshape(1, n, 1, 256)), to_dev(xb[1].reshape(1, n, 1, 256)),
                        to_dev(np.zeros(1, np.int32)))
    kc, ks = oracle.q8_quantize_vectors(xb[0])
    vc, vs = oracle.q8_quantize_vectors(xb[1])
    torch.cuda.synchronize()
    for name, want in (("k_codes", kc), ("v_codes", vc), ("k_scales", ks), ("v_scales", vs)):
        g = host_plane(gc, name)
        bad = np.nonzero(np.any(g != want, axis=-1))[0]
        assert bad.size == 0, f"{name}: {bad.size} rows differ, first {bad[:5]}"


# ------------------------------------------------------------------ decode
def build_contig(seed, B, H, T, dt="bf16", outliers=16.0):
    k, v = synth.kv_tokens(seed, B, T, H, 256, 0.01, outliers)
    if dt == "bf16":
        k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.contiguous(B, H, T, bits=8)
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T, bits=8)
    sp = np.zeros(B, np.int32)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(sp))
    oc.append(k, v, sp)
    return gc, oc, k, v


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_decode_group_sizes(G):
    B, H, T = 2, 2, 700
    gc, oc, _, _ = build_contig(280 + G, B, H, T)
    q = synth.to_bf16_bits(synth.queries(280 + G, B, H * G, 256))
    lens = np.array([700, 333], np.int32)
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    want = oc.decode_attn(q, lens, 1 / 16)
    compare_cache(gc, oc)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("qdt", ["bf16", "f32"])
def test_decode_tile_boundaries(qdt):
    """Lengths around the 64-token tile and the 16-token warp slices, several
    splits per sequence."""
    lens = np.array([1, 15, 16, 17, 63, 64, 65, 200, 1023, 2049, 5000], np.int32)
    B, H, G, T = len(lens), 1, 8, 5000
    gc, oc, _, _ = build_contig(295, B, H, T)
    q = synth.queries(296, B, H * G, 256)
    if qdt == "bf16":
        q = synth.to_bf16_bits(q)
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 0.0625).cpu().numpy()
    want = oc.decode_attn(q, lens, 0.0625)
    assert np.abs(got - want).max() <= ATOL


def test_decode_outlier_query_and_zero_query():
    """Near one-hot softmax (x20 outlier channels in q, K and V) and an
    all-zero query head (uniform weights: the mean of V)."""
    ch = np.array(synth.WORKLOADS["tiny"]["outlier_channels"])
    k = synth.apply_outliers(synth.gaussian(2110, (1, 512, 1, 256)), ch, 20.0)
    v = synth.apply_outliers(synth.gaussian(2120, (1, 512, 1, 256)), ch, 20.0)
    gc = kvq.Q4Cache.contiguous(1, 1, 512, bits=8)
    oc = oracle.Q4Cache(512, 1, max_tokens=512, bits=8)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(1, np.int32)))
    oc.append(k, v, np.zeros(1, np.int32))
    q = synth.apply_outliers(synth.gaussian(2130, (1, 4, 256)), ch, 20.0)
    q[0, 2] = 0.0
    got = kvq.decode_attn(gc, to_dev(q), to_dev(np.array([512], np.int32)), 512, 1 / 16).cpu().numpy()
    want = oc.decode_attn(q, [512], 1 / 16)
    assert np.abs(got - want).max() <= ATOL


def test_decode_zero_and_clamped_lengths():
    B, H, T = 3, 1, 300
    gc, oc, _, _ = build_contig(290, B, H, T)
    q = synth.to_bf16_bits(synth.queries(290, B, 8, 256))
    lens = np.array([0, 300, 1000], np.int32)
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), 300, 0.0625).cpu().numpy()
    want = oc.decode_attn(q, np.minimum(lens, 300), 0.0625)
    assert np.all(got[0] == 0)
    assert np.abs(got - want).max() <= ATOL


def test_decode_paged_equals_contiguous_and_oracle():
    B, H, G, ps = 4, 2, 8, 64
    lens = np.array([64, 777, 5, 1200], np.int32)
    T = int(lens.max())
    bt, n_pages = paged_setup(211, B, lens, ps)
    k = synth.to_bf16_bits(synth.gaussian(291, (B, T, H, 256)))
    v = synth.to_bf16_bits(synth.gaussian(292, (B, T, H, 256)))
    q = synth.to_bf16_bits(synth.queries(293, B, H * G, 256))
    pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), bits=8)
    cc = kvq.Q4Cache.contiguous(B, H, T, bits=8)
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps, bits=8)
    append_paged(pc, oc, k, v, lens, bt)
    kvq.quantize_append(cc, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    gp = kvq.decode_attn(pc, to_dev(q), to_dev(lens), T, 0.0625).cpu().numpy()
    gcn = kvq.decode_attn(cc, to_dev(q), to_dev(lens), T, 0.0625).cpu().numpy()
    want = oc.decode_attn(q, lens, 0.0625)
    assert np.abs(gp - want).max() <= ATOL
    np.testing.assert_array_equal(gp, gcn)


def test_decode_unmapped_pages_contribute_nothing():
    B, H, G, ps = 2, 2, 4, 64
    lens = np.array([640, 300], np.int32)
    T = int(lens.max())
    bt, n_pages = paged_setup(213, B, lens, ps)
    k = synth.to_bf16_bits(synth.gaussian(295, (B, T, H, 256)))
    v = synth.to_bf16_bits(synth.gaussian(296, (B, T, H, 256)))
    q = synth.to_bf16_bits(synth.queries(297, B, H * G, 256))
    pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), bits=8)
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps, bits=8)
    append_paged(pc, oc, k, v, lens, bt)
    holes = bt.copy()
    holes[0, 3] = -1
    holes[0, 6] = n_pages + 2
    holes[1, 1] = -1
    got = kvq.decode_attn(pc.with_block_table(torch.from_numpy(holes)), to_dev(q),
                          to_dev(lens), T, 0.0625).cpu().numpy()
    compact = np.full_like(bt, -1)
    keep0 = [j for j in range(10) if j not in (3, 6)]
    keep1 = [j for j in range(5) if j != 1]
    compact[0, :len(keep0)] = bt[0, keep0]
    compact[1, :len(keep1)] = bt[1, keep1]
    clens = np.array([640 - 2 * ps, 300 - ps], np.int32)
    want = oc.with_block_table(compact).decode_attn(q, clens, 0.0625)
    assert np.abs(got - want).max() <= ATOL


# ------------------------------------------------------------------ step, multi
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_step_equals_append_then_decode(dt):
    B, H, G, T = 3, 2, 8, 1500
    pos = np.array([1000, 37, 1499], np.int32)
    k, v = synth.kv_tokens(300, B, T, H, 256, 0.01, 16.0)
    nk, nv = synth.kv_tokens(302, B, 1, H, 256, 0.01, 16.0)
    q = synth.queries(301, B, H * G, 256)
    cvt = synth.to_bf16_bits if dt == "bf16" else (lambda x: x)
    k, v, q = cvt(k), cvt(v), cvt(q)
    nk, nv = np.ascontiguousarray(cvt(nk)[:, 0]), np.ascontiguousarray(cvt(nv)[:, 0])
    base = kvq.Q4Cache.contiguous(B, H, T, bits=8)
    kvq.quantize_append(base, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    a = kvq.Q4Cache.contiguous(B, H, T, bits=8)
    f = kvq.Q4Cache.contiguous(B, H, T, bits=8)
    for name in PLANES:
        getattr(a, name).copy_(getattr(base, name))
        getattr(f, name).copy_(getattr(base, name))
    kvq.quantize_append(a, to_dev(nk[:, None]), to_dev(nv[:, None]), to_dev(pos))
    want_gpu = kvq.decode_attn(a, to_dev(q), to_dev(pos + 1), T, 1 / 16)
    got = kvq.decode_step(f, to_dev(nk), to_dev(nv), to_dev(q), to_dev(pos), T, 1 / 16)
    torch.cuda.synchronize()
    for name in PLANES:
        assert torch.equal(getattr(f, name), getattr(a, name)), name
    assert torch.equal(got, want_gpu)
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T, bits=8)
    oc.append(k, v, np.zeros(B, np.int32))
    oc.append(nk[:, None], nv[:, None], pos)
    assert np.abs(got.cpu().numpy() - oc.decode_attn(q, pos + 1, 1 / 16)).max() <= ATOL


def test_multi_token_decode():
    B, H, G, T = 3, 2, 4, 800
    gc, oc, _, _ = build_contig(510, B, H, T)
    q_to_seq = np.array([0, 0, 0, 1, 2, 2, 5], np.int32)
    q_lens = np.array([798, 799, 800, 300, 1, 64, 100], np.int32)
    q = synth.to_bf16_bits(synth.queries(520, len(q_to_seq), H * G, 256))
    got = kvq.decode_attn_multi(gc, to_dev(q), to_dev(q_to_seq), to_dev(q_lens), B, T,
                                1 / 16).cpu().numpy()
    for i in range(len(q_to_seq)):
        s = int(q_to_seq[i])
        if s >= B:
            assert not np.any(got[i])
            continue
        qb = np.zeros((B,) + q.shape[1:], q.dtype)
        qb[s] = q[i]
        lens = np.zeros(B, np.int32)
        lens[s] = q_lens[i]
        assert np.abs(got[i] - oc.decode_attn(qb, lens, 1 / 16)[s]).max() <= ATOL


# ------------------------------------------------------------------ full size
def test_long_decode_q8_full_size_sampled():
    """The long-context shape (1 x 131072 tokens, 32 q / 4 kv heads, bf16)
    over a Q8_0 cache: sampled rows bit-exact, all 32 head outputs within 2e-3."""
    W = synth.WORKLOADS["long_decode"]
    B, H, T, Hq = W["batch"], W["n_kv_heads"], W["ctx"], W["n_q_heads"]
    k, v = synth.kv_tokens(W["seed"], B, T, H, 256, W["outlier_frac"], W["outlier_factor"])
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    q = synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256))
    gc = kvq.Q4Cache.contiguous(B, H, T, bits=8)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    got = kvq.decode_attn(gc, to_dev(q), to_dev(np.array([T], np.int32)), T, 1 / 16).cpu().numpy()
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T, bits=8)
    oc.append(k, v, np.zeros(B, np.int32))
    rng = np.random.default_rng(0)
    compare_cache(gc, oc, rows=rng.choice(B * H * T, 4096, replace=False))
    assert np.abs(got - oc.decode_attn(q, [T], 1 / 16)).max() <= ATOL
