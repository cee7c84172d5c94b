"""Pins for the oracle's rotation (fwht_blocks) and its fp16 converter.

Each pin comes from outside the oracle: a hand-derived golden case, the
explicit Sylvester matrix, closed forms, or numpy's float16 conversion.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _hexf(h):
    return np.array([int(x, 16) for x in h], np.uint32).view(np.float32)


def sylvester(n):
    """Explicit Hadamard matrix H[i][j] = (-1)^popcount(i & j) / sqrt(n), fp64."""
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0) / np.sqrt(n)


def test_stage_order_golden():
    g = json.load(open(os.path.join(GOLD, "fwht_stage_order.json")))
    x = _hexf(g["input_hex_f32"])
    y = oracle.fwht_f32(x, block=g["block"])
    assert y.view(np.uint32).tolist() == _hexf(g["expected_hex_f32"]).view(np.uint32).tolist()
    # the golden discriminates: the other stage order is a different answer
    assert g["expected_hex_f32"] != g["reverse_order_hex_f32"]


def test_end_scaling_block128():
    # x = [1, 3, 0, ...]: every stage is exact on small integers, giving +4 / -2
    # patterns; the single end multiply by fp32(1/sqrt(128)) is then exact too.
    x = np.zeros(128, np.float32)
    x[0], x[1] = 1.0, 3.0
    y = oracle.fwht_f32(x, block=128)
    s = np.float32(1.0 / np.sqrt(128.0))
    want = (sylvester(128) * np.sqrt(128.0)) @ x.astype(np.float64)
    np.testing.assert_array_equal(y, (want.astype(np.float32) * s).astype(np.float32))
    assert set(np.unique(want)) == {-2.0, 4.0}


@pytest.mark.parametrize("block", [4, 64, 128, 256])
def test_matches_sylvester_bruteforce(block):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 256)).astype(np.float32)
    H = sylvester(block)
    ref = np.concatenate([x[:, b:b + block].astype(np.float64) @ H.T
                          for b in range(0, 256, block)], axis=1)
    y32 = oracle.fwht_f32(x, block=block)
    y64 = oracle.fwht_f64(x.astype(np.float64), block=block)
    np.testing.assert_allclose(y64, ref, rtol=0, atol=1e-12)
    # fp32 butterflies: log2(block) roundings of magnitude <= |x|_1-ish
    np.testing.assert_allclose(y32, ref, rtol=0, atol=2e-5 * np.abs(x).max() * np.log2(block))


def test_closed_forms_256():
    e0 = np.zeros(256, np.float32)
    e0[0] = 1.0
    np.testing.assert_array_equal(oracle.fwht_f32(e0), np.full(256, 0.0625, np.float32))
    ones = np.ones(256, np.float32)
    want = np.zeros(256, np.float32)
    want[0] = 16.0
    np.testing.assert_array_equal(oracle.fwht_f32(ones), want)


def test_self_inverse_and_dot_invariance():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 256))
    np.testing.assert_allclose(oracle.fwht_f64(oracle.fwht_f64(x)), x, atol=1e-12)
    x32 = x.astype(np.float32)
    np.testing.assert_allclose(oracle.fwht_f32(oracle.fwht_f32(x32)), x32, atol=5e-6)
    q, k = rng.standard_normal((2, 64, 256))
    hq, hk = oracle.fwht_f64(q), oracle.fwht_f64(k)
    lhs = np.sum(hq * hk, axis=1)
    rhs = np.sum(q * k, axis=1)
    # <Hq, Hk> == <q, k> to 1e-5 relative (Strata PR #21, How 3)
    assert np.all(np.abs(lhs - rhs) <= 1e-5 * np.sqrt(np.sum(q * q, 1) * np.sum(k * k, 1)))


def test_f16_converter_against_numpy():
    # every 2^-13-th fp32 bit pattern plus the boundary region of every exponent
    rng = np.random.default_rng(0)
    pats = [np.arange(0, 1 << 32, 8191, dtype=np.uint64)]
    for e in range(100, 145):  # around the binary16 range, subnormals included
        base = np.uint64(e << 23)
        pats.append(base + rng.integers(0, 1 << 23, 20000).astype(np.uint64))
        pats.append(base + (np.arange(-64, 64, dtype=np.int64).astype(np.uint64) + np.uint64(0x1000)) % np.uint64(1 << 23))
    u = np.concatenate(pats).astype(np.uint32)
    u = np.concatenate([u, u | np.uint32(0x80000000)])
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    got = oracle.f32_to_f16_bits(f)
    with np.errstate(over="ignore"):
        want = f.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_f16_converter_exhaustive():
    """Every one of the 2^32 fp32 bit patterns converts exactly as numpy's
    round-to-nearest-even binary16 conversion does (NaN payloads excepted:
    non-finite input is outside the quantizers' contract).  Chunks of 2^24
    patterns run on all host cores (numpy's cast and the ctypes call release
    the GIL)."""
    import ctypes as C
    from concurrent.futures import ThreadPoolExecutor

    L = oracle.lib()
    n = 1 << 24

    def sweep(chunks):
        base = np.arange(n, dtype=np.uint32)
        u = np.empty(n, np.uint32)
        want = np.empty(n, np.float16)
        got = np.empty(n, np.uint16)
        f = u.view(np.float32)
        bad = 0
        with np.errstate(over="ignore", invalid="ignore"):
            for c in chunks:
                np.add(base, np.uint32(c * n), out=u)
                np.copyto(want, f, casting="unsafe")
                L.orc_f32_to_f16_array(f.ctypes.data_as(C.c_void_p),
                                       got.ctypes.data_as(C.c_void_p), C.c_int64(n))
                diff = want.view(np.uint16) != got
                if diff.any():
                    bad += int((diff & ~np.isnan(f)).sum())
        return bad

    k = os.cpu_count() or 1
    with ThreadPoolExecutor(k) as ex:
        assert sum(ex.map(sweep, [range(i, 256, k) for i in range(k)])) == 0


def test_f16_roundtrip_exact():
    h = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    h = h[np.isfinite(h.view(np.float16))]
    f = oracle.f16_bits_to_f32(h)
    np.testing.assert_array_equal(f, h.view(np.float16).astype(np.float32))
