"""Pins of the oracle's Q8_0 + FWHT-256 variant (the 8-bit KV cache the pages
compare Q4_0 against), by hand-derived blocks, closed forms, invariances, the
rounding bound and a brute-force attention over an explicit Hadamard matrix."""
import numpy as np
import pytest

import oracle
from hadamard_rotated_bit_fwht_b200 import synth


def test_hand_built_block_halves_away_from_zero():
    # amax 127 -> d = 1 exactly, id = 1: codes are the values rounded half away
    z = np.zeros(32, np.float32)
    z[:8] = [127, -63.5, 0.5, -0.5, 1.5, -2.5, 126.49, -0.49]
    qs, d = oracle.q8_0_block(z)
    assert d == 0x3C00  # fp16(1.0)
    assert list(qs[:8]) == [127, -64, 1, -1, 2, -3, 126, 0]
    assert not np.any(qs[8:])


def test_zero_block_and_negative_amax():
    qs, d = oracle.q8_0_block(np.zeros(32, np.float32))
    assert d == 0 and not np.any(qs)
    z = np.zeros(32, np.float32)
    z[3], z[4] = -254.0, 3.0  # amax 254 from a negative value -> d = 2
    qs, d = oracle.q8_0_block(z)
    assert d == 0x4000  # fp16(2.0)
    assert qs[3] == -127 and qs[4] == 2  # 3 / 2 = 1.5 -> 2


def test_sign_symmetry_and_power_of_two_scaling():
    g = np.random.default_rng(3)
    for _ in range(200):
        z = (g.standard_normal(32) * g.uniform(0.01, 100)).astype(np.float32)
        qs, d = oracle.q8_0_block(z)
        qn, dn = oracle.q8_0_block(-z)
        assert np.array_equal(qn, -qs) and dn == d
        q2, d2 = oracle.q8_0_block(z * np.float32(4))
        assert np.array_equal(q2, qs)
        assert oracle.f16_bits_to_f32(np.array([d2], np.uint16))[0] == \
            4 * oracle.f16_bits_to_f32(np.array([d], np.uint16))[0]


def test_max_code_and_rounding_bound():
    """The max-abs element codes to +-127; every element is within half a step
    (amax / 254) plus the fp16 rounding of the scale (127 codes x 2^-11 d)."""
    g = np.random.default_rng(4)
    for _ in range(500):
        z = (g.standard_normal(32) * g.uniform(1e-3, 1e3)).astype(np.float32)
        z[g.integers(32)] *= 8  # an outlier
        qs, d = oracle.q8_0_block(z)
        amax = float(np.abs(z).max())
        j = int(np.argmax(np.abs(z)))
        assert abs(int(qs[j])) == 127
        back = oracle.q8_0_dequant_block(qs, d)
        err = np.abs(back - z.astype(np.float64)).max()
        assert err <= amax / 254 * (1 + 1e-6) + amax * 2.0 ** -11


def test_fwht_lowers_int8_error_on_outlier_channels():
    """The pages' quality claim for int8 (rel-L2 drops with the rotation on data
    with outlier channels); checked qualitatively on seeded data."""
    x = synth.gaussian(77, (512, 256))
    x[:, [5, 100, 200]] *= 20
    codes, scales = oracle.q8_quantize_vectors(x)
    rot = oracle.fwht_f32(x)
    err_rot = []
    err_plain = []
    for i in range(64):
        rec = np.concatenate([oracle.q8_0_dequant_block(codes[i, 32 * b:32 * b + 32], scales[i, b])
                              for b in range(8)])
        err_rot.append(np.linalg.norm(rec - rot[i]) / np.linalg.norm(rot[i]))
        plain = []
        for b in range(8):
            q, d = oracle.q8_0_block(x[i, 32 * b:32 * b + 32])
            plain.append(oracle.q8_0_dequant_block(q, d))
        plain = np.concatenate(plain)
        err_plain.append(np.linalg.norm(plain - x[i]) / np.linalg.norm(x[i]))
    assert np.mean(err_rot) < np.mean(err_plain)


def hadamard256():
    i = np.arange(256)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2, -1.0, 1.0) / 16.0


def test_attention_brute_force():
    """Attention over a Q8_0 cache equals softmax attention over the rows
    dequantized and rotated back with an explicit Hadamard matrix."""
    B, H, G, T = 2, 1, 4, 48
    k = synth.gaussian(81, (B, T, H, 256))
    v = synth.gaussian(82, (B, T, H, 256))
    q = synth.gaussian(83, (B, H * G, 256))
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T, bits=8)
    oc.append(k, v, np.zeros(B, np.int32))
    lens = np.array([48, 17], np.int32)
    got = oc.decode_attn(q, lens, 0.0625)
    Hm = hadamard256()
    for b in range(B):
        rows = [b * T + t for t in range(lens[b])]

        def deq(codes, scales):
            r = np.stack([np.concatenate([oracle.q8_0_dequant_block(codes[x, 32 * j:32 * j + 32],
                                                                    scales[x, j])
                                          for j in range(8)]) for x in rows])
            return r @ Hm  # H is symmetric: rows back to the original basis
        kk, vv = deq(oc.k_codes, oc.k_scales), deq(oc.v_codes, oc.v_scales)
        for h in range(H * G):
            s = 0.0625 * kk @ q[b, h].astype(np.float64)
            p = np.exp(s - s.max())
            p /= p.sum()
            assert np.allclose(got[b, h], p @ vv, atol=1e-12, rtol=1e-9)


@pytest.mark.parametrize("bad", [np.nan, np.inf])
def test_non_finite_rejected(bad):
    z = np.zeros(32, np.float32)
    z[1] = bad
    with pytest.raises(ValueError):
        oracle.q8_0_block(z)
