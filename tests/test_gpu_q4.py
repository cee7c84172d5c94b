"""GPU parity of the Q4_0 + FWHT-256 path against the CPU oracle, through the
C ABI.  Rotation, codes and scales must be bit-identical; attention must be
within 2e-3 max-abs of the oracle's fp64 evaluation of the same cache."""
import numpy as np
import pytest
import torch

import oracle
from hadamard_rotated_bit_fwht_b200 import build, kvq, synth

pytestmark = pytest.mark.gpu
ATOL = 2e-3  # attention tolerance (max-abs vs the fp64 oracle)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    kvq.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda() if dtype is None else t.to(dtype).cuda()


# ------------------------------------------------------------------ rotate
@pytest.mark.parametrize("n_vec", [1, 3, 16, 17, 1000, 4099])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_rotate_bitexact(n_vec, dt):
    x = synth.gaussian(50 + n_vec, (n_vec, 256)) * np.float32(3)
    x[:, 7] *= 20
    if dt == "bf16":
        xb = synth.to_bf16_bits(x)
        want = oracle.fwht_f32(synth.bf16_bits_to_f32(xb))
        got = kvq.rotate(to_dev(xb)).cpu().numpy()
    else:
        want = oracle.fwht_f32(x)
        got = kvq.rotate(to_dev(x)).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_rotate_empty():
    x = torch.empty((0, 256), device="cuda")
    assert kvq.rotate(x).shape == (0, 256)


# ------------------------------------------------------------------ append
def compare_cache(gpu: kvq.Q4Cache, orc: oracle.Q4Cache, rows=None):
    for name in ("k_codes", "v_codes", "k_scales", "v_scales"):
        g = getattr(gpu, name).cpu().numpy()
        o = getattr(orc, name)
        if name.endswith("scales"):
            g = g.view(np.uint16)
        if rows is not None:
            g, o = g[rows], o[rows]
        mism = np.nonzero(np.any(g != o, axis=-1))[0]
        assert mism.size == 0, f"{name}: {mism.size} rows differ, first {mism[:5]}"


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_append_tiny_contiguous(dt):
    """Tiny workload: 1 sequence, 1 kv head, 512 tokens, fp32 with four x20
    outlier channels; quantized in three appends (prefill, chunk, single)."""
    W = synth.WORKLOADS["tiny"]
    k = synth.gaussian(W["seed"] * 1000 + 10, (1, 512, 1, 256))
    v = synth.gaussian(W["seed"] * 1000 + 20, (1, 512, 1, 256))
    ch = np.array(W["outlier_channels"])
    k = synth.apply_outliers(k, ch, W["outlier_factor"])
    v = synth.apply_outliers(v, ch, W["outlier_factor"])
    if dt == "bf16":
        k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.contiguous(1, 1, 512)
    oc = oracle.Q4Cache(512, 1, max_tokens=512)
    for lo, hi in [(0, 300), (300, 511), (511, 512)]:
        sp = np.array([lo], np.int32)
        kvq.quantize_append(gc, to_dev(k[:, lo:hi]), to_dev(v[:, lo:hi]), to_dev(sp))
        oc.append(k[:, lo:hi], v[:, lo:hi], sp)
    torch.cuda.synchronize()
    compare_cache(gc, oc)


def test_append_ragged_batch_and_skip():
    """Several sequences at different start positions; positions beyond the
    capacity are skipped and rows before the start positions stay untouched."""
    B, H, T, cap = 3, 5, 37, 64
    k = synth.to_bf16_bits(synth.gaussian(61, (B, T, H, 256)) * 4)
    v = synth.to_bf16_bits(synth.gaussian(62, (B, T, H, 256)))
    sp = np.array([0, 20, 40], np.int32)  # sequence 2 runs past position 63
    gc = kvq.Q4Cache.contiguous(B, H, cap)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(sp))
    torch.cuda.synchronize()
    g = {n: getattr(gc, n).cpu().numpy() for n in ("k_codes", "v_codes", "k_scales", "v_scales")}
    for b in range(B):
        n = min(T, cap - int(sp[b]))
        one = oracle.Q4Cache(H * cap, H, max_tokens=cap)
        one.append(k[b:b + 1, :n], v[b:b + 1, :n], sp[b:b + 1])
        for h in range(H):
            base_g, base_o = (b * H + h) * cap, h * cap
            for name in g:
                got = g[name][base_g:base_g + cap]
                if name.endswith("scales"):
                    got = got.view(np.uint16)
                want = getattr(one, name)[base_o:base_o + cap]
                assert np.array_equal(got, want), (b, h, name)


def paged_setup(seed, B, H, lens, ps, extra=3):
    """Shuffled page table; unused columns are -1 (never reached)."""
    npp = [(int(L) + ps - 1) // ps for L in lens]
    maxp = max(npp) + 1
    bt, n_pages = synth.page_table(seed, B, np.array(npp), maxp, extra_pages=extra)
    return bt, n_pages


def append_paged(gpu, orc, k, v, lens, bt):
    """Append sequence b's first lens[b] tokens, one sequence at a time."""
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
    bt, n_pages = paged_setup(9, B, H, lens, ps)
    k = synth.to_bf16_bits(synth.gaussian(71, (B, T, H, 256)) * 2)
    v = synth.to_bf16_bits(synth.gaussian(72, (B, T, H, 256)))
    gc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    append_paged(gc, oc, k, v, lens, bt)
    torch.cuda.synchronize()
    compare_cache(gc, oc)


def test_append_stress_bitexact():
    """One million rotated vectors with magnitudes spread over six decades and
    outlier channels: every code and scale bit-identical to the oracle.  (This
    size exposes a contracted multiply-add, which changes about one code in a
    million.)"""
    n = 1 << 20
    x = synth.gaussian(123, (2, n, 256))
    mag = np.exp(np.random.default_rng(5).uniform(np.log(1e-3), np.log(1e3), (2, n, 1))).astype(np.float32)
    x = (x * mag).astype(np.float32)
    x[:, ::17, 200] *= 30
    xb = synth.to_bf16_bits(x)
    k = xb[0].reshape(1, n, 1, 256)
    v = xb[1].reshape(1, n, 1, 256)
    gc = kvq.Q4Cache.contiguous(1, 1, n)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(1, np.int32)))
    kc, ks = oracle.q4_quantize_vectors(xb[0])
    vc, vs = oracle.q4_quantize_vectors(xb[1])
    torch.cuda.synchronize()
    for got, want in ((gc.k_codes, kc), (gc.v_codes, vc), (gc.k_scales, ks), (gc.v_scales, vs)):
        g = got.cpu().numpy()
        if g.dtype == np.int16:
            g = g.view(np.uint16)
        bad = np.nonzero(np.any(g != want, axis=-1))[0]
        assert bad.size == 0, f"{bad.size} rows differ, first {bad[:5]}"


# ------------------------------------------------------------------ decode
def build_contig(seed, B, H, T, dt="bf16", outliers=16.0):
    k, v = synth.kv_tokens(seed, B, T, H, 256, 0.01, outliers)
    if dt == "bf16":
        k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.contiguous(B, H, T)
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T)
    sp = np.zeros(B, np.int32)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(sp))
    oc.append(k, v, sp)
    return gc, oc


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_decode_group_sizes(G):
    B, H, T = 2, 2, 700
    gc, oc = build_contig(80 + G, B, H, T)
    q = synth.to_bf16_bits(synth.queries(80 + G, B, H * G, 256))
    lens = np.array([700, 333], np.int32)
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 1 / 16).cpu().numpy()
    want = oc.decode_attn(q, lens, 1 / 16)
    compare_cache(gc, oc)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("qdt", ["bf16", "f32"])
def test_decode_tile_boundaries(qdt):
    """Lengths around the 64-token tile and 16-token warp slices, several
    splits per sequence, fp32 and bf16 queries."""
    lens = np.array([1, 15, 16, 63, 64, 65, 200, 1023, 2049, 5000], np.int32)
    B, H, G, T = len(lens), 1, 8, 5000
    gc, oc = build_contig(95, B, H, T)
    q = synth.queries(96, B, H * G, 256)
    if qdt == "bf16":
        q = synth.to_bf16_bits(q)
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), T, 0.0625).cpu().numpy()
    want = oc.decode_attn(q, lens, 0.0625)
    assert np.abs(got - want).max() <= ATOL


def test_decode_tiny_workload():
    """Tiny workload end to end: fp32 K, V, q with four x20 outlier channels
    (near one-hot softmax), and a second query without outliers."""
    W = synth.WORKLOADS["tiny"]
    ch = np.array(W["outlier_channels"])
    k = synth.apply_outliers(synth.gaussian(1010, (1, 512, 1, 256)), ch, 20.0)
    v = synth.apply_outliers(synth.gaussian(1020, (1, 512, 1, 256)), ch, 20.0)
    gc = kvq.Q4Cache.contiguous(1, 1, 512)
    oc = oracle.Q4Cache(512, 1, max_tokens=512)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(1, np.int32)))
    oc.append(k, v, np.zeros(1, np.int32))
    q_out = synth.apply_outliers(synth.gaussian(1030, (1, 4, 256)), ch, 20.0)
    q_plain = synth.gaussian(1031, (1, 4, 256))
    for q in (q_out, q_plain):
        got = kvq.decode_attn(gc, to_dev(q), to_dev(np.array([512], np.int32)), 512,
                              1 / 16).cpu().numpy()
        want = oc.decode_attn(q, [512], 1 / 16)
        assert np.abs(got - want).max() <= ATOL


def test_decode_zero_and_clamped_lengths():
    B, H, T = 3, 1, 300
    gc, oc = build_contig(90, B, H, T)
    q = synth.to_bf16_bits(synth.queries(90, B, 8, 256))
    lens = np.array([0, 300, 1000], np.int32)  # 1000 is clamped to max_seq_len = 300
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), 300, 0.0625).cpu().numpy()
    want = oc.decode_attn(q, np.minimum(lens, 300), 0.0625)
    assert np.all(got[0] == 0)
    assert np.abs(got - want).max() <= ATOL


def test_decode_paged_equals_contiguous_and_oracle():
    B, H, G, ps = 4, 2, 8, 64
    lens = np.array([64, 777, 5, 1200], np.int32)
    T = int(lens.max())
    bt, n_pages = paged_setup(11, B, H, lens, ps)
    k = synth.to_bf16_bits(synth.gaussian(91, (B, T, H, 256)))
    v = synth.to_bf16_bits(synth.gaussian(92, (B, T, H, 256)))
    q = synth.to_bf16_bits(synth.queries(93, B, H * G, 256))
    sp = np.zeros(B, np.int32)
    pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    cc = kvq.Q4Cache.contiguous(B, H, T)
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    append_paged(pc, oc, k, v, lens, bt)
    kvq.quantize_append(cc, to_dev(k), to_dev(v), to_dev(sp))
    gp = kvq.decode_attn(pc, to_dev(q), to_dev(lens), T, 0.0625).cpu().numpy()
    gcn = kvq.decode_attn(cc, to_dev(q), to_dev(lens), T, 0.0625).cpu().numpy()
    want = oc.decode_attn(q, lens, 0.0625)
    assert np.abs(gp - want).max() <= ATOL
    np.testing.assert_array_equal(gp, gcn)  # same tokens, same splits -> same bits


def test_decode_unmapped_pages_contribute_nothing():
    """Page-table entries that name no page (-1, or past the pool) drop their
    tokens; with no positional term in decode attention the result equals the
    oracle over the table with those pages removed."""
    B, H, G, ps = 2, 2, 4, 64
    lens = np.array([640, 300], np.int32)
    T = int(lens.max())
    bt, n_pages = paged_setup(13, B, H, lens, ps)
    k = synth.to_bf16_bits(synth.gaussian(95, (B, T, H, 256)))
    v = synth.to_bf16_bits(synth.gaussian(96, (B, T, H, 256)))
    q = synth.to_bf16_bits(synth.queries(97, B, H * G, 256))
    pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
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


# ------------------------------------------------------------------ full size
def test_long_decode_full_size_sampled():
    """Long-context workload at full size (1 x 131072 tokens, 32 q / 4 kv
    heads, bf16) through the call the benchmark times: kvq_decode_step with
    the cache holding the first 131071 tokens and the new token appended at
    position 131071 by the split that holds it.  The appended rows and
    sampled other rows bit-exact, all 32 head outputs within 2e-3."""
    W = synth.WORKLOADS["long_decode"]
    B, H, T, Hq = W["batch"], W["n_kv_heads"], W["ctx"], W["n_q_heads"]
    k, v = synth.kv_tokens(W["seed"], B, T, H, 256, W["outlier_frac"], W["outlier_factor"])
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    q = synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256))
    gc = kvq.Q4Cache.contiguous(B, H, T)
    kvq.quantize_append(gc, to_dev(k[:, :T - 1]), to_dev(v[:, :T - 1]),
                        to_dev(np.zeros(B, np.int32)))
    got = kvq.decode_step(gc, to_dev(k[:, T - 1]), to_dev(v[:, T - 1]), to_dev(q),
                          to_dev(np.full(B, T - 1, np.int32)), T, 1 / 16).cpu().numpy()
    threads = oracle.host_threads()
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T)
    oc.append(k, v, np.zeros(B, np.int32), threads=threads)
    rng = np.random.default_rng(0)
    new_rows = [(b * H + h) * T + T - 1 for b in range(B) for h in range(H)]
    compare_cache(gc, oc, rows=np.concatenate([new_rows, rng.choice(B * H * T, 4096, replace=False)]))
    want = oc.decode_attn(q, [T], 1 / 16, threads=threads)
    assert np.abs(got - want).max() <= ATOL


def test_long_decode_longest_context():
    """One sequence of 524288 tokens (4x the long-context workload; 32 q / 4
    kv heads, bf16, the workload's outlier channels): the decode sums 4x more
    tokens per split, so an error that grows with the summed tokens shows
    here.  Sampled cache rows bit-exact, all 32 head outputs within 2e-3."""
    W = synth.WORKLOADS["long_decode"]
    B, H, Hq, T = 1, W["n_kv_heads"], W["n_q_heads"], 524288
    k, v = synth.kv_tokens(W["seed"] + T, B, T, H, 256, W["outlier_frac"], W["outlier_factor"])
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    q = synth.to_bf16_bits(synth.queries(W["seed"] + T, B, Hq, 256))
    gc = kvq.Q4Cache.contiguous(B, H, T)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    got = kvq.decode_attn(gc, to_dev(q), to_dev(np.full(B, T, np.int32)), T, 1 / 16).cpu().numpy()
    threads = oracle.host_threads()
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T)
    oc.append(k, v, np.zeros(B, np.int32), threads=threads)
    rng = np.random.default_rng(1)
    compare_cache(gc, oc, rows=rng.choice(B * H * T, 4096, replace=False))
    want = oc.decode_attn(q, [T], 1 / 16, threads=threads)
    assert np.abs(got - want).max() <= ATOL


def test_quantize_workload_full_size():
    """Quantize-on-append workload at full size (8 sequences x 8 kv heads,
    bf16): a 4096-token prefill, then 256 single-token appends, as the
    benchmark drives them; every code and scale row bit-identical to the
    oracle quantising all 4352 tokens at once."""
    W = synth.WORKLOADS["quantize"]
    B, H, P, A, cap = W["batch"], W["n_kv_heads"], W["prefill"], W["appends"], W["capacity"]
    k, v = synth.kv_tokens(W["seed"], B, P + A, H, 256, W["outlier_frac"], W["outlier_factor"])
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    del k, v
    gc = kvq.Q4Cache.contiguous(B, H, cap)
    kvq.quantize_append(gc, to_dev(kb[:, :P]), to_dev(vb[:, :P]), to_dev(np.zeros(B, np.int32)))
    for i in range(A):
        kvq.quantize_append(gc, to_dev(kb[:, P + i:P + i + 1]), to_dev(vb[:, P + i:P + i + 1]),
                            to_dev(np.full(B, P + i, np.int32)))
    oc = oracle.Q4Cache(B * H * cap, H, max_tokens=cap)
    oc.append(kb, vb, np.zeros(B, np.int32))
    torch.cuda.synchronize()
    compare_cache(gc, oc)


def test_paged_decode_full_size():
    """Batched paged workload at full size (32 sequences of U[8192, 32768]
    tokens, 16 q / 2 kv heads, 256-token shuffled pages, bf16) in the launch
    configuration the benchmark times (the balanced stream schedule over all
    64 units): every output row of all 32 sequences within 2e-3 of the oracle
    and every cache row bit-identical (the oracle runs its (sequence, kv head)
    units on all host cores)."""
    W = synth.WORKLOADS["paged_decode"]
    B, H, Hq, ps = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["page_size"]
    lens = synth.seq_lens(W["seed"], B, W["ctx_lo"], W["ctx_hi"])
    npp = (lens + ps - 1) // ps
    bt, n_pages = synth.page_table(W["seed"], B, npp, int(npp.max()))
    gc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    threads = oracle.host_threads()
    for b0 in range(0, B, 8):  # the benchmark's generation: 8 sequences at a time
        Lc = int(lens[b0:b0 + 8].max())
        k, v = synth.kv_tokens(W["seed"] * 100 + b0, 8, Lc, H, 256, W["outlier_frac"],
                               W["outlier_factor"])
        kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
        del k, v
        for j in range(8):
            b, L = b0 + j, int(lens[b0 + j])
            kvq.quantize_append(gc.with_block_table(torch.from_numpy(bt[b:b + 1])),
                                to_dev(kb[j:j + 1, :L]), to_dev(vb[j:j + 1, :L]),
                                to_dev(np.zeros(1, np.int32)))
            oc.with_block_table(bt[b:b + 1]).append(kb[j:j + 1, :L], vb[j:j + 1, :L],
                                                    np.zeros(1, np.int32), threads=threads)
        del kb, vb
    q = synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256))
    got = kvq.decode_attn(gc, to_dev(q), to_dev(lens), int(lens.max()), 1 / 16).cpu().numpy()
    compare_cache(gc, oc)
    want = oc.decode_attn(q, lens, 1 / 16, threads=threads)
    err = np.abs(got - want).max(axis=(1, 2))
    assert err.max() <= ATOL, f"sequences over 2e-3: {np.nonzero(err > ATOL)[0]}"
