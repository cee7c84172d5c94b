"""Pins for the oracle's Q4_0 decode attention (Strata PR #21: What (score
invariance), How 2, merge note (per-token path rotates Q and the output);
vLLM rocm_octave reference_attention for the GQA / zero-length semantics)."""
import numpy as np
import pytest

import oracle
from hadamard_rotated_bit_fwht_b200 import synth
from test_oracle_fwht import sylvester

H256 = sylvester(256)


def np_dequant_rows(codes, scales):
    """Independent dequantization: nibble extraction + numpy float16."""
    lo = (codes & 15).astype(np.float64) - 8
    hi = (codes >> 4).astype(np.float64) - 8
    d = scales.view(np.float16).astype(np.float64)  # (n, 8)
    vals = np.empty(codes.shape[:-1] + (256,), np.float64)
    for b in range(8):
        vals[..., b * 32:b * 32 + 16] = lo[..., b * 16:(b + 1) * 16] * d[..., b:b + 1]
        vals[..., b * 32 + 16:b * 32 + 32] = hi[..., b * 16:(b + 1) * 16] * d[..., b:b + 1]
    return vals


def build(seed, B, Hkv, Hq, T, outliers=True, dtype="bf16"):
    k, v = synth.kv_tokens(seed, B, T, Hkv, 256, 0.01, 16.0 if outliers else 1.0)
    q = synth.queries(seed, B, Hq, 256)
    if dtype == "bf16":
        k, v, q = synth.to_bf16_bits(k), synth.to_bf16_bits(v), synth.to_bf16_bits(q)
    cache = oracle.Q4Cache(B * Hkv * T, Hkv, max_tokens=T)
    cache.append(k, v, np.zeros(B, np.int32))
    return cache, q


def brute_force(cache, q, seq_lens, scale):
    B, Hq, _ = q.shape
    Hkv = cache.n_kv_heads
    G = Hq // Hkv
    qf = q.astype(np.float64) if q.dtype == np.float32 else synth.bf16_bits_to_f32(q).astype(np.float64)
    out = np.zeros((B, Hq, 256))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            L = seq_lens[b]
            if L <= 0:
                continue
            rows = (b * Hkv + g) * cache.max_tokens + np.arange(L)
            K = np_dequant_rows(cache.k_codes[rows], cache.v_scales[rows] * 0 + cache.k_scales[rows]) @ H256.T
            V = np_dequant_rows(cache.v_codes[rows], cache.v_scales[rows]) @ H256.T
            s = scale * (K @ qf[b, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            out[b, h] = p @ V
    return out


def test_bruteforce_tiny():
    cache, q = build(21, B=2, Hkv=2, Hq=8, T=48)
    sl = np.array([48, 17], np.int32)
    got = cache.decode_attn(q, sl, 1 / 16)
    want = brute_force(cache, q, sl, 1 / 16)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_rotated_space_identity():
    """Scores in the rotated space with q_rot = H q and the output rotated back
    once per head equal attention in the original basis."""
    cache, q = build(22, B=1, Hkv=1, Hq=4, T=64, dtype="f32")
    got = cache.decode_attn(q, [64], 0.0625)
    Kr = np_dequant_rows(cache.k_codes[:64], cache.k_scales[:64])
    Vr = np_dequant_rows(cache.v_codes[:64], cache.v_scales[:64])
    for h in range(4):
        qr = H256 @ q[0, h].astype(np.float64)
        s = 0.0625 * (Kr @ qr)
        p = np.exp(s - s.max())
        p /= p.sum()
        o = H256 @ (p @ Vr)
        np.testing.assert_allclose(got[0, h], o, atol=1e-12)


def test_uniform_scores_give_mean_value():
    T = 40
    k = np.zeros((1, T, 1, 256), np.float32)  # all-zero K -> zero scores
    v = synth.gaussian(5, (1, T, 1, 256))
    cache = oracle.Q4Cache(T, 1, max_tokens=T)
    cache.append(k, v, [0])
    q = synth.gaussian(6, (1, 2, 256))
    got = cache.decode_attn(q, [T], 0.1)
    Vr = np_dequant_rows(cache.v_codes, cache.v_scales) @ H256.T
    for h in range(2):
        np.testing.assert_allclose(got[0, h], Vr.mean(0), atol=1e-12)


def test_zero_length_and_gqa_mapping():
    B, Hkv, Hq, T = 3, 2, 6, 16
    k = np.zeros((B, T, Hkv, 256), np.float32)
    # constant value vector per kv head: V[b, :, g] = (g + 1) * e_j pattern
    v = np.zeros((B, T, Hkv, 256), np.float32)
    for g in range(Hkv):
        v[:, :, g, :] = (g + 1) * synth.gaussian(40 + g, (256,))
    cache = oracle.Q4Cache(B * Hkv * T, Hkv, max_tokens=T)
    cache.append(k, v, np.zeros(B, np.int32))
    q = synth.gaussian(7, (B, Hq, 256))
    out = cache.decode_attn(q, [T, 0, 5], 1.0)
    assert np.all(out[1] == 0.0)
    G = Hq // Hkv
    for b in (0, 2):
        for h in range(Hq):
            g = h // G
            row = (b * Hkv + g) * T
            want = np_dequant_rows(cache.v_codes[row:row + 1], cache.v_scales[row:row + 1])[0] @ H256.T
            np.testing.assert_allclose(out[b, h], want, atol=1e-12)


def test_paged_equals_contiguous():
    B, Hkv, Hq, T, ps = 2, 2, 4, 70, 16
    k = synth.to_bf16_bits(synth.gaussian(8, (B, T, Hkv, 256)))
    v = synth.to_bf16_bits(synth.gaussian(9, (B, T, Hkv, 256)))
    q = synth.to_bf16_bits(synth.gaussian(10, (B, Hq, 256)))
    cc = oracle.Q4Cache(B * Hkv * T, Hkv, max_tokens=T)
    cc.append(k, v, [0, 0])
    npp = (T + ps - 1) // ps
    bt, n_pages = synth.page_table(3, B, np.array([npp, npp]), npp + 1, extra_pages=3)
    pc = oracle.Q4Cache(n_pages * Hkv * ps, Hkv, block_table=bt, page_size=ps)
    pc.append(k, v, [0, 0])
    sl = [70, 33]
    np.testing.assert_array_equal(cc.decode_attn(q, sl, 0.0625), pc.decode_attn(q, sl, 0.0625))


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("bits", [4, 8])
def test_threaded_units_bit_identical(paged, bits):
    """The threaded harness (independent (sequence, kv head) decode units and
    (sequence, token chunk) append units of the unchanged C oracle) gives
    exactly the single-call results."""
    B, Hkv, Hq, T, ps = 3, 2, 8, 300, 64
    k, v = synth.kv_tokens(77, B, T, Hkv, 256, 0.01, 16.0)
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    q = synth.to_bf16_bits(synth.queries(78, B, Hq, 256))
    lens = np.array([300, 0, 129], np.int32)
    if paged:
        npp = -(-T // ps)
        bt, n_pages = synth.page_table(79, B, np.full(B, npp), npp)

        def mk():
            return oracle.Q4Cache(n_pages * Hkv * ps, Hkv, block_table=bt, page_size=ps, bits=bits)
    else:
        def mk():
            return oracle.Q4Cache(B * Hkv * T, Hkv, max_tokens=T, bits=bits)
    one, many = mk(), mk()
    one.append(kb, vb, np.zeros(B, np.int32))
    many.append(kb, vb, np.zeros(B, np.int32), threads=4, chunk=37)
    for a in ("k_codes", "k_scales", "v_codes", "v_scales"):
        assert np.array_equal(getattr(one, a), getattr(many, a)), a
    want = one.decode_attn(q, lens, 1 / 16)
    got = one.decode_attn(q, lens, 1 / 16, threads=4)
    assert np.array_equal(got, want)


def test_threaded_octave_bit_identical():
    fmt = (128, 64, 4, 0)
    s = synth.sign_pattern(128)
    nblk, Hkv, Hq, bs = 8, 2, 8, 16
    k = synth.to_bf16_bits(synth.gaussian(21, (nblk * bs, Hkv, 128)))
    v = synth.to_bf16_bits(synth.gaussian(22, (nblk * bs, Hkv, 128)))
    slots = oracle.octave_quantize(k, v, fmt, s)
    assert np.array_equal(oracle.octave_quantize(k, v, fmt, s, threads=3, chunk=10), slots)
    cache = slots.reshape(nblk, bs, Hkv, 128).transpose(0, 2, 1, 3).copy()
    bt = np.array([[5, 2, 7, 0], [1, 3, 4, 6]], np.int32)
    q = synth.to_bf16_bits(synth.gaussian(23, (3, Hq, 128)))
    q2r = np.array([0, 1, 1], np.int32)
    q2l = np.array([50, 64, 0], np.int32)
    want = oracle.octave_attention(q, cache, bt, q2r, q2l, fmt, 0.09, s)
    got = oracle.octave_attention(q, cache, bt, q2r, q2l, fmt, 0.09, s, threads=3)
    assert np.array_equal(got, want)
