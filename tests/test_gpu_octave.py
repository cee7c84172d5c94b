"""GPU parity of the Octave variant (vLLM rocm_octave page) against the CPU
oracle through the C ABI: slots bit-identical, attention within 2e-3."""
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


def to_dev(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def make_cache(fmt, T, Hkv, bs, seed, dt="bf16", outliers=16.0, shuffle=True):
    """T tokens into ceil(T / bs) + 2 blocks through a shuffled slot mapping."""
    nblk = (T + bs - 1) // bs + 2
    k = synth.apply_outliers(synth.gaussian(seed, (T, Hkv, 128)),
                             synth.outlier_channels(seed, Hkv, 128), outliers)
    v = synth.apply_outliers(synth.gaussian(seed + 1, (T, Hkv, 128)),
                             synth.outlier_channels(seed, Hkv, 128), outliers)
    if dt == "bf16":
        k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    g = np.random.default_rng(seed)
    blocks = g.permutation(nblk) if shuffle else np.arange(nblk)
    slot = (blocks[np.arange(T) // bs] * bs + np.arange(T) % bs).astype(np.int64)
    return k, v, slot, nblk


@pytest.mark.parametrize("v_bits", [4, 3])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_quantize_bitexact(v_bits, dt):
    fmt = (128, 64, v_bits, 0)
    F = kvq.OctaveFormat(*fmt[:3])
    slot_bytes = F.layout()["slot_bytes"]
    T, Hkv, bs = 333, 3, 16
    k, v, slot, nblk = make_cache(fmt, T, Hkv, bs, 7 + v_bits, dt)
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, slot_bytes), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(k), to_dev(v), to_dev(slot), cache, kvq.sign_words(signs))
    want = oracle.octave_quantize(k, v, fmt, signs)  # (T, H, slot)
    got = cache.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, Hkv, slot_bytes)[slot]
    bad = np.nonzero(np.any(got != want, axis=-1))
    assert bad[0].size == 0, f"{bad[0].size} slots differ, first token {bad[0][:3]}"


@pytest.mark.parametrize("T,Hkv", [(1, 1), (3, 1), (5, 3), (7, 5)])
@pytest.mark.parametrize("fmt", [(128, 64, 4, 0), (128, 64, 3, 1)])
def test_quantize_few_items_bitexact(T, Hkv, fmt):
    """Item counts that leave octets of the last warp without an item (the
    kernel runs eight threads per (token, kv head) and whole warps together)."""
    F = kvq.OctaveFormat(fmt[0], fmt[1], fmt[2], compact=bool(fmt[3]))
    slot_bytes = F.layout()["slot_bytes"]
    bs = 4
    k, v, slot, nblk = make_cache(fmt, T, Hkv, bs, 90 + T * Hkv, "bf16")
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, slot_bytes), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(k), to_dev(v), to_dev(slot), cache, kvq.sign_words(signs))
    want = oracle.octave_quantize(k, v, fmt, signs)
    c = cache.cpu().numpy()
    got = c.transpose(0, 2, 1, 3).reshape(-1, Hkv, slot_bytes)[slot]
    assert np.array_equal(got, want)
    # slots no token maps to stay untouched
    used = np.zeros(nblk * bs, bool)
    used[slot] = True
    assert not c.transpose(0, 2, 1, 3).reshape(-1, Hkv, slot_bytes)[~used].any()


def test_quantize_skips_negative_and_out_of_range_slots():
    F = kvq.OctaveFormat(128, 64, 4)
    T, Hkv, bs = 8, 2, 16
    k, v, slot, nblk = make_cache((128, 64, 4, 0), T, Hkv, bs, 3, shuffle=False)
    slot[2] = -1
    slot[5] = nblk * bs + 3  # block out of range
    cache = torch.zeros((nblk, Hkv, bs, 128), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(k), to_dev(v), to_dev(slot), cache,
                        kvq.sign_words(synth.sign_pattern(128)))
    c = cache.cpu().numpy()
    assert np.all(c[0, :, 2] == 0) and np.all(c[0, :, 5] == 0)
    assert np.any(c[0, :, 3] != 0)


def decode_case(v_bits, G, bs, qdt, seed=21):
    """Requests over a shuffled block mapping; returns what both sides need."""
    fmt = (128, 64, v_bits, 0)
    F = kvq.OctaveFormat(128, 64, v_bits)
    slot_bytes = F.layout()["slot_bytes"]
    Hkv = 2
    Hq = Hkv * G
    T = 600
    k, v, slot, nblk = make_cache(fmt, T, Hkv, bs, seed)
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, slot_bytes), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(k), to_dev(v), to_dev(slot), cache, kvq.sign_words(signs))
    # request r owns the blocks holding tokens [192 r, 192 r + 192)
    nreq, span = 3, 192
    maxb = -(-span // bs)
    bt = np.zeros((nreq, maxb), np.int32)
    for r in range(nreq):
        for j in range(maxb):
            bt[r, j] = slot[min(span * r + j * bs, T - 1)] // bs
    q = synth.queries(seed + 10, 4, Hq, 128)
    if qdt == "bf16":
        q = synth.to_bf16_bits(q)
    return F, fmt, cache, bt, q, signs


@pytest.mark.parametrize("v_bits", [4, 3])  # 4: tensor-core kernel, 3: SIMT kernel
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("qdt", ["bf16", "f32"])
def test_decode_vs_oracle(v_bits, G, qdt):
    F, fmt, cache, bt, q, signs = decode_case(v_bits, G, 16, qdt)
    q_to_req = np.array([0, 1, 2, 0], np.int32)
    q_to_klen = np.array([192, 45, 0, 129], np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q), cache, to_dev(bt), to_dev(q_to_req),
                                 to_dev(q_to_klen), 192, 128 ** -0.5,
                                 kvq.sign_words(signs)).cpu().numpy()
    want = oracle.octave_attention(q, cache.cpu().numpy(), bt, q_to_req, q_to_klen, fmt,
                                   128 ** -0.5, signs)
    assert np.all(got[2] == 0)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("v_bits", [4, 3])
@pytest.mark.parametrize("bs", [1, 24, 64, 256])
def test_decode_block_sizes(v_bits, bs):
    """Block sizes below, across and above the 64-token tile."""
    F, fmt, cache, bt, q, signs = decode_case(v_bits, 4, bs, "bf16", seed=40 + bs)
    q_to_req = np.array([2, 0, 1, 1], np.int32)
    q_to_klen = np.array([192, 191, 65, 1], np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q), cache, to_dev(bt), to_dev(q_to_req),
                                 to_dev(q_to_klen), 192, 128 ** -0.5,
                                 kvq.sign_words(signs)).cpu().numpy()
    want = oracle.octave_attention(q, cache.cpu().numpy(), bt, q_to_req, q_to_klen, fmt,
                                   128 ** -0.5, signs)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("v_bits,bs", [(4, 16), (3, 16), (4, 64)])
def test_decode_unmapped_blocks_contribute_nothing(v_bits, bs):
    """A block-table entry that names no block (-1 or past the cache) drops its
    tokens: decode attention has no positional term, so the result equals the
    oracle over the table with those entries removed.  (64-token blocks take
    the tensor-copy staging, whole tiles at a time.)"""
    F, fmt, cache, bt, q, signs = decode_case(v_bits, 8, bs, "bf16", seed=60)
    nblk = cache.shape[0]
    holes = bt.copy()
    nb = bt.shape[1]
    gone0 = (1, 2) if nb < 8 else (3, 7)
    holes[0, gone0[0]] = -1
    holes[0, gone0[1]] = nblk + 5
    holes[1, 0] = -1
    keep0 = [j for j in range(nb) if j not in gone0]
    keep1 = [j for j in range(nb) if j != 0]
    q_to_req = np.array([0, 1], np.int32)
    q_to_klen = np.array([192, 192], np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q[:2]), cache, to_dev(holes), to_dev(q_to_req),
                                 to_dev(q_to_klen), 192, 128 ** -0.5,
                                 kvq.sign_words(signs)).cpu().numpy()
    c = cache.cpu().numpy()
    for i, keep in enumerate((keep0, keep1)):
        compact = bt[i, keep][None, :]
        want = oracle.octave_attention(q[i:i + 1], c, compact, np.zeros(1, np.int32),
                                       np.array([bs * len(keep)], np.int32), fmt,
                                       128 ** -0.5, signs)
        assert np.abs(got[i:i + 1] - want).max() <= ATOL


def test_octave_workload_full_size():
    """Octave workload at the benchmark's own shape and inputs (k3v4, head
    128, rope 64, 16 requests x 16384 tokens, 32 q / 8 kv heads, bf16,
    256-token shuffled blocks, the same per-request generation): every slot
    bit-exact and all 16 x 32 head outputs within 2e-3 of the oracle (which
    runs token chunks and query tokens on all host cores)."""
    W = synth.WORKLOADS["octave"]
    fmt = (W["head_size"], W["rope_dim"], W["v_bits"], 0)
    F = kvq.OctaveFormat(*fmt[:3])
    B, Hkv, Hq, ctx, bs = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["ctx"], W["block_size"]
    bt, _ = synth.page_table(W["seed"], B, np.full(B, ctx // bs), ctx // bs)
    signs = synth.sign_pattern(128)
    cache = torch.zeros((B * ctx // bs, Hkv, bs, 128), dtype=torch.uint8, device="cuda")
    threads = oracle.host_threads()
    nblk = B * ctx // bs
    want_by_slot = np.zeros((nblk * bs, Hkv, 128), np.uint8)
    for r in range(B):
        k, v = synth.kv_tokens(W["seed"] * 100 + r, 1, ctx, Hkv, 128, W["outlier_frac"],
                               W["outlier_factor"])
        kb, vb = synth.to_bf16_bits(k[0]), synth.to_bf16_bits(v[0])
        del k, v
        slot = (bt[r, np.arange(ctx) // bs] * bs + np.arange(ctx) % bs).astype(np.int64)
        kvq.octave_quantize(F, to_dev(kb), to_dev(vb), to_dev(slot), cache, kvq.sign_words(signs))
        slots = oracle.octave_quantize(kb, vb, fmt, signs, threads=threads)  # (ctx, Hkv, 128)
        want_by_slot[slot] = slots
    got_by_slot = cache.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, Hkv, 128)
    bad = np.nonzero(np.any(got_by_slot != want_by_slot, axis=-1))
    assert bad[0].size == 0, f"{bad[0].size} slots differ"
    # the oracle attends over its own cache, in the (blocks, kv heads, block, slot) layout
    want_cache = want_by_slot.reshape(nblk, bs, Hkv, 128).transpose(0, 2, 1, 3).copy()
    q = synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 128))
    q_to_req = np.arange(B, dtype=np.int32)
    q_to_klen = np.full(B, ctx, np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q), cache, to_dev(bt), to_dev(q_to_req),
                                 to_dev(q_to_klen), ctx, 128 ** -0.5,
                                 kvq.sign_words(signs)).cpu().numpy()
    want = oracle.octave_attention(q, want_cache, bt, q_to_req, q_to_klen, fmt, 128 ** -0.5,
                                   signs, threads=threads)
    err = np.abs(got - want).max(axis=(1, 2))
    assert err.max() <= ATOL, f"requests over 2e-3: {np.nonzero(err > ATOL)[0]}"


def test_octave_decode_longest_context():
    """One request of 262144 tokens (1024 shuffled 256-token blocks, 8 kv
    heads, GQA 4, the workload's outlier channels): the k3v4 decode sums 16x
    more tokens per request than the benchmark workload, so an error that
    grows with the summed tokens shows here.  Slots bit-exact, all 32 head
    outputs within 2e-3 of the oracle over the oracle's own slots."""
    W = synth.WORKLOADS["octave"]
    fmt = (128, 64, 4, 0)
    F = kvq.OctaveFormat(*fmt[:3])
    Hkv, Hq, ctx, bs, seed = 8, 32, 262144, 256, 31
    nblk = ctx // bs
    bt, _ = synth.page_table(seed, 1, np.array([nblk]), nblk)
    signs = synth.sign_pattern(128)
    k, v = synth.kv_tokens(seed, 1, ctx, Hkv, 128, W["outlier_frac"], W["outlier_factor"])
    kb, vb = synth.to_bf16_bits(k[0]), synth.to_bf16_bits(v[0])
    del k, v
    slot = (bt[0, np.arange(ctx) // bs] * bs + np.arange(ctx) % bs).astype(np.int64)
    cache = torch.zeros((nblk, Hkv, bs, 128), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(kb), to_dev(vb), to_dev(slot), cache, kvq.sign_words(signs))
    threads = oracle.host_threads()
    want_by_slot = np.zeros((nblk * bs, Hkv, 128), np.uint8)
    want_by_slot[slot] = oracle.octave_quantize(kb, vb, fmt, signs, threads=threads)
    got_by_slot = cache.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, Hkv, 128)
    assert np.array_equal(got_by_slot, want_by_slot)
    want_cache = want_by_slot.reshape(nblk, bs, Hkv, 128).transpose(0, 2, 1, 3).copy()
    q = synth.to_bf16_bits(synth.queries(seed, 1, Hq, 128))
    q_to_req = np.zeros(1, np.int32)
    q_to_klen = np.full(1, ctx, np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q), cache, to_dev(bt), to_dev(q_to_req),
                                 to_dev(q_to_klen), ctx, 128 ** -0.5,
                                 kvq.sign_words(signs)).cpu().numpy()
    want = oracle.octave_attention(q, want_cache, bt, q_to_req, q_to_klen, fmt, 128 ** -0.5,
                                   signs, threads=threads)
    err = np.abs(got - want).max()
    assert err <= ATOL, f"max abs error {err}"


@pytest.mark.parametrize("v_bits,bs", [(4, 256), (4, 16), (3, 16)])
def test_decode_right_after_quantize_sees_the_new_slots(v_bits, bs):
    """Append and decode back to back on one stream with every input already
    on the device, so no copy or synchronisation separates the two launches
    (on the tensor-core path the decode and its combine are programmatic
    dependent launches): four rounds, each appending 200 tokens to each of 2
    requests and decoding over everything so far, must see every slot the
    append before them wrote.  All outputs within 2e-3 of the oracle."""
    fmt = (128, 64, v_bits, 0)
    F = kvq.OctaveFormat(128, 64, v_bits)
    sbytes = F.layout()["slot_bytes"]
    Hkv, G, R, step, rounds = 2, 4, 2, 200, 4
    T = step * rounds
    per_req = -(-T // bs)
    nblk = R * per_req + 3
    blocks = np.random.default_rng(bs).permutation(nblk)[:R * per_req].reshape(R, per_req)
    bt = blocks.astype(np.int32)
    signs = synth.sign_pattern(128)
    k, v = synth.kv_tokens(919, R, T, Hkv, 128, 0.01, 16.0)
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    t = np.arange(T)
    slot = np.stack([bt[r, t // bs].astype(np.int64) * bs + t % bs for r in range(R)])
    q = synth.to_bf16_bits(synth.queries(920, rounds * R, Hkv * G, 128))
    # every round's inputs staged on the device before the first launch
    chunks = [(to_dev(kb[:, i * step:(i + 1) * step].reshape(-1, Hkv, 128)),
               to_dev(vb[:, i * step:(i + 1) * step].reshape(-1, Hkv, 128)),
               to_dev(slot[:, i * step:(i + 1) * step].reshape(-1)),
               to_dev(q[i * R:(i + 1) * R]),
               to_dev(np.full(R, (i + 1) * step, np.int32))) for i in range(rounds)]
    bt_d, q2r_d = to_dev(bt), to_dev(np.arange(R, dtype=np.int32))
    sw = kvq.sign_words(signs)
    cache = torch.zeros((nblk, Hkv, bs, sbytes), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    outs = []
    for kc, vc, sc, qc, lc in chunks:
        kvq.octave_quantize(F, kc, vc, sc, cache, sw)
        outs.append(kvq.octave_decode_attn(F, qc, cache, bt_d, q2r_d, lc, T, 128 ** -0.5, sw))
    got = [o.cpu().numpy() for o in outs]
    want_slots = oracle.octave_quantize(kb.reshape(-1, Hkv, 128), vb.reshape(-1, Hkv, 128), fmt,
                                        signs)
    oc = np.zeros((nblk * bs, Hkv, sbytes), np.uint8)
    oc[slot.reshape(-1)] = want_slots
    oc = oc.reshape(nblk, bs, Hkv, sbytes).transpose(0, 2, 1, 3).copy()
    for i in range(rounds):
        want = oracle.octave_attention(q[i * R:(i + 1) * R], oc, bt, np.arange(R, dtype=np.int32),
                                       np.full(R, (i + 1) * step, np.int32), fmt, 128 ** -0.5,
                                       signs)
        err = np.abs(got[i] - want).max()
        assert err <= ATOL, f"round {i}: max abs error {err}"


# ------------------------------------------------------------------ compact K
@pytest.mark.parametrize("v_bits", [3, 4])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_compact_quantize_bitexact(v_bits, dt):
    """Compact K (octave_k3v3_compact and its 4-bit-V sibling): one whole-head
    rotation of K with 3-bit codes and a single scale; 4-byte slot padding."""
    fmt = (128, 64, v_bits, 1)
    F = kvq.OctaveFormat(128, 64, v_bits, True)
    slot_bytes = F.layout()["slot_bytes"]
    T, Hkv, bs = 257, 2, 16
    k, v, slot, nblk = make_cache(fmt, T, Hkv, bs, 90 + v_bits, dt)
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, slot_bytes), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(k), to_dev(v), to_dev(slot), cache, kvq.sign_words(signs))
    want = oracle.octave_quantize(k, v, fmt, signs)
    got = cache.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, Hkv, slot_bytes)[slot]
    bad = np.nonzero(np.any(got != want, axis=-1))
    assert bad[0].size == 0, f"{bad[0].size} slots differ, first token {bad[0][:3]}"


@pytest.mark.parametrize("v_bits", [3, 4])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_compact_decode_vs_oracle(v_bits, G):
    fmt = (128, 64, v_bits, 1)
    F = kvq.OctaveFormat(128, 64, v_bits, True)
    slot_bytes = F.layout()["slot_bytes"]
    Hkv, bs, T = 2, 16, 600
    k, v, slot, nblk = make_cache(fmt, T, Hkv, bs, 95 + G)
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, slot_bytes), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(k), to_dev(v), to_dev(slot), cache, kvq.sign_words(signs))
    nreq, span = 3, 192
    maxb = -(-span // bs)
    bt = np.zeros((nreq, maxb), np.int32)
    for r in range(nreq):
        for j in range(maxb):
            bt[r, j] = slot[min(span * r + j * bs, T - 1)] // bs
    q = synth.to_bf16_bits(synth.queries(97 + G, 4, Hkv * G, 128))
    q_to_req = np.array([0, 1, 2, 0], np.int32)
    q_to_klen = np.array([192, 45, 0, 129], np.int32)
    got = kvq.octave_decode_attn(F, to_dev(q), cache, to_dev(bt), to_dev(q_to_req),
                                 to_dev(q_to_klen), 192, 128 ** -0.5,
                                 kvq.sign_words(signs)).cpu().numpy()
    want = oracle.octave_attention(q, cache.cpu().numpy(), bt, q_to_req, q_to_klen, fmt,
                                   128 ** -0.5, signs)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("fmt", [(128, 64, 4, 0), (128, 64, 3, 0), (128, 0, 4, 0),
                                 (128, 128, 3, 0), (128, 64, 3, 1), (128, 64, 4, 1)],
                         ids=lambda f: "-".join(map(str, f)))
def test_quantize_stress_bitexact(fmt):
    """2^20 (token, head) vectors for k3v4 (2^16 for the other formats) whose
    magnitudes span 2^-40 .. 2^40 per vector, with exact zeros, repeated
    values and single spikes mixed in: every slot bit-identical to the oracle.
    The kernel takes codes from a floor table of 2 y except within 2^-13 of a
    doubled midpoint, where it redoes the IEEE division; this drives both
    paths and the zero / tiny-vector cases."""
    n_tok, Hkv = (131072, 8) if fmt == (128, 64, 4, 0) else (8192, 8)
    F = kvq.OctaveFormat(128, fmt[1], fmt[2], bool(fmt[3]))
    slot_bytes = F.layout()["slot_bytes"]
    rng = np.random.default_rng(sum(fmt) + fmt[1])
    k = synth.gaussian(900 + fmt[2], (n_tok, Hkv, 128))
    v = synth.gaussian(901 + fmt[2], (n_tok, Hkv, 128))
    scale = np.exp2(rng.integers(-40, 41, size=(n_tok, Hkv, 1))).astype(np.float32)
    k *= scale
    v *= scale[::-1]
    k[rng.random((n_tok, Hkv)) < 0.002] = 0.0          # all-zero vectors
    v[rng.random((n_tok, Hkv, 128)) < 0.01] = 0.0      # scattered exact zeros
    rep = rng.random((n_tok, Hkv)) < 0.01              # constant vectors
    k[rep] = np.float32(1.5)
    spike = rng.random((n_tok, Hkv)) < 0.01            # one large element
    k[spike, 3] *= np.float32(1e4)
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    slot = np.arange(n_tok, dtype=np.int64)
    bs = 256
    nblk = n_tok // bs
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, slot_bytes), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, to_dev(kb), to_dev(vb), to_dev(slot), cache, kvq.sign_words(signs))
    want = oracle.octave_quantize(kb, vb, fmt, signs, threads=oracle.host_threads())
    got = cache.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, Hkv, slot_bytes)
    bad = np.nonzero(np.any(got != want, axis=-1))
    assert bad[0].size == 0, f"{bad[0].size} slots differ, first (token, head) {list(zip(*bad))[:3]}"


def test_quantize_rejects_misaligned_inputs():
    F = kvq.OctaveFormat(128, 64, 4)
    k = torch.zeros(2 * 128 * 2 + 8, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((1, 2, 16, 128), dtype=torch.uint8, device="cuda")
    slot = torch.zeros(1, dtype=torch.int64, device="cuda")
    kk = k[4:4 + 256].view(1, 2, 128)  # 8 bytes past a 16-byte boundary
    with pytest.raises(kvq.KVQError) as e:
        kvq.octave_quantize(F, kk, kk, slot, cache, kvq.sign_words(synth.sign_pattern(128)))
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


def test_bindings_refuse_a_cache_of_another_slot_width():
    """The C ABI takes the slot width from the format, so the bindings check
    the cache's last dimension against it: a k3v3 format (112-byte slots)
    with a 128-byte-slot cache is refused before any launch."""
    F = kvq.OctaveFormat(128, 64, 3)
    assert F.layout()["slot_bytes"] == 112
    cache = torch.zeros((1, 2, 16, 128), dtype=torch.uint8, device="cuda")
    k = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    signs = kvq.sign_words(synth.sign_pattern(128))
    with pytest.raises(ValueError):
        kvq.octave_quantize(F, k, k, torch.zeros(1, dtype=torch.int64, device="cuda"), cache,
                            signs)
    i32 = lambda *v: torch.tensor(v, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        kvq.octave_decode_attn(F, torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda"),
                               cache, torch.zeros((1, 1), dtype=torch.int32, device="cuda"),
                               i32(0), i32(16), 16, 0.1, signs)
    torch.cuda.synchronize()
    assert not cache.any().item()
