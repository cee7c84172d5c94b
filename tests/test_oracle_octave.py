"""Pins for the oracle's Octave variant (vLLM API page
'vllm.v1.attention.ops.rocm_octave': OctaveFormat, _pack, _quantize_lut,
fwht_blocks, reference_quantize / reference_dequantize / reference_attention,
v_block) and its Lloyd-Max N(0,1) codebook (textbook: Max 1960)."""
import json
import os

import numpy as np
import pytest
from scipy import stats

import oracle
from hadamard_rotated_bit_fwht_b200 import synth
from test_oracle_fwht import sylvester

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FMT = (128, 64, 4, 0)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLD, "octave_format.json")))["cases"],
                         ids=lambda c: str(c["fmt"]))
def test_format_offsets(case):
    f = oracle.octave_format(*case["fmt"])
    for key in ("off_k_nope", "off_v", "off_scales", "num_scales", "slot_bytes", "kernel_code"):
        assert f[key] == case[key], key


def test_format_validation():
    with pytest.raises(ValueError):
        oracle.octave_format(128, 64, 5)          # V bits must be 3 or 4
    with pytest.raises(ValueError):
        oracle.octave_format(192, 64, 3, True)    # compact needs a power-of-two head
    with pytest.raises(ValueError):
        oracle.octave_format(128, 32, 4)          # rope not a multiple of 64


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLD, "octave_pack.json")))["cases"],
                         ids=lambda c: str(c["bits"]))
def test_pack_golden(case):
    codes = np.array(case["codes"] if "codes" in case else [d % 8 for d in range(32)], np.uint8)
    packed = oracle.octave_pack(codes, case["bits"])
    assert packed.tobytes().hex() == case["packed_hex"]
    np.testing.assert_array_equal(oracle.octave_unpack(packed, codes.size, case["bits"]), codes)


@pytest.mark.parametrize("bits,n", [(4, 64), (4, 128), (3, 64), (3, 128)])
def test_pack_roundtrip_and_plane_rules(bits, n):
    rng = np.random.default_rng(bits * n)
    codes = rng.integers(0, 1 << bits, n).astype(np.uint8)
    p = oracle.octave_pack(codes, bits)
    assert p.size == n * bits // 8
    np.testing.assert_array_equal(oracle.octave_unpack(p, n, bits), codes)
    words = p.view("<u4")
    if bits == 4:  # w & 0x0F0F0F0F / (w >> 4) & 0x0F0F0F0F give dims 0..3 / 4..7
        for w in range(n // 8):
            lo = (words[w] & 0x0F0F0F0F).tobytes()
            hi = ((words[w] >> 4) & 0x0F0F0F0F).tobytes()
            assert list(lo) == codes[8 * w:8 * w + 4].tolist()
            assert list(hi) == codes[8 * w + 4:8 * w + 8].tolist()
    else:
        lo_w, hi_w = words[:n // 16], words[n // 16:]
        for d in range(n):
            i2, j = (d % 16) // 4, d % 4
            l2 = (int(lo_w[d // 16]) >> (2 * i2)) & 0x03030303
            i1 = (d % 32) // 4
            h1 = (int(hi_w[d // 32]) >> i1) & 0x01010101
            assert ((l2 >> (8 * j)) & 0xFF) + 4 * ((h1 >> (8 * j)) & 0xFF) == codes[d]


@pytest.mark.parametrize("bits", [3, 4])
def test_lloyd_max_textbook(bits):
    g = json.load(open(os.path.join(GOLD, "lloyd_max_n01.json")))
    c, b = oracle.lloyd_max(bits)
    pos = g["levels_8_positive" if bits == 3 else "levels_16_positive"]
    np.testing.assert_allclose(c[len(c) // 2:], pos, atol=g["tolerance"])
    np.testing.assert_allclose(c, -c[::-1], atol=1e-12)  # symmetric
    # optimality, checked with scipy's normal distribution (independent code):
    edges = np.concatenate([[-np.inf], b, [np.inf]])
    for i in range(len(c)):
        lo, hi = edges[i], edges[i + 1]
        mass = stats.norm.cdf(hi) - stats.norm.cdf(lo)
        mean = (stats.norm.pdf(lo) - stats.norm.pdf(hi)) / mass
        assert abs(mean - c[i]) < 1e-9
    np.testing.assert_allclose(b, (c[1:] + c[:-1]) / 2, atol=1e-15)


@pytest.mark.parametrize("bits", [3, 4])
def test_codebook_int8(bits):
    lut, mult = oracle.octave_codebook(bits)
    c, _ = oracle.lloyd_max(bits)
    assert lut[-1] == 127 and lut[0] == -127
    assert np.all(np.diff(lut.astype(int)) > 0)
    assert mult == np.float32(127.0 / c[-1])
    np.testing.assert_array_equal(lut, np.round(c * (127.0 / c[-1])).astype(np.int8))


@pytest.mark.parametrize("bits,n", [(4, 64), (3, 64), (4, 128)])
def test_quantize_lut_norm_preserving(bits, n):
    rng = np.random.default_rng(bits + n)
    lut, _ = oracle.octave_codebook(bits)
    for _ in range(200):
        x = (rng.standard_normal(n) * rng.uniform(0.01, 20)).astype(np.float32)
        codes, s = oracle.octave_quantize_lut(x, bits)
        s16 = np.float32(s).astype(np.float16).astype(np.float64)
        xhat = lut[codes].astype(np.float64) * s16 / 64.0
        ss = np.dot(x.astype(np.float64), x.astype(np.float64))
        # x . x_hat = |x|^2 up to the fp16 rounding of the scale (and fp32 sums)
        assert abs(np.dot(x, xhat) - ss) <= (2.0 ** -11 + 1e-5) * ss


def test_quantize_lut_zero_block():
    codes, s = oracle.octave_quantize_lut(np.zeros(64, np.float32), 4)
    assert s == 0.0


def test_rotate_unrotate():
    rng = np.random.default_rng(1)
    s = synth.sign_pattern(128)
    x = rng.standard_normal(128).astype(np.float32)
    for block in (64, 128):
        y = oracle.octave_rotate(x, s, block)
        H = sylvester(block)
        want = np.concatenate([H @ (x * s)[i:i + block].astype(np.float64) for i in range(0, 128, block)])
        np.testing.assert_allclose(y, want, atol=1e-5)
        np.testing.assert_allclose(oracle.octave_unrotate(y, s, block), x, atol=1e-5)


def test_quantize_dequantize_roundtrip_quality():
    T, H = 64, 4
    s = synth.sign_pattern(128)
    k = synth.gaussian(3, (T, H, 128))
    v = synth.gaussian(4, (T, H, 128))
    slots = oracle.octave_quantize(k, v, FMT, s)
    assert slots.shape == (T, H, 128) and np.all(slots[..., 126:] == 0)  # pad bytes are zero
    kh, vh = oracle.octave_dequantize(slots, FMT, s)
    rel_k = np.linalg.norm(kh - k) / np.linalg.norm(k)
    rel_v = np.linalg.norm(vh - v) / np.linalg.norm(v)
    assert rel_k < 0.2 and rel_v < 0.15  # 3/4-bit Lloyd-Max on Gaussians
    # rotated=True keeps the rotated basis: rotating it back gives the same K, V
    kr, vr = oracle.octave_dequantize(slots, FMT, s, rotated=True)
    for t in range(T):
        for h in range(H):
            np.testing.assert_allclose(oracle.octave_unrotate(kr[t, h], s, 64), kh[t, h], atol=1e-12)
            np.testing.assert_allclose(oracle.octave_unrotate(vr[t, h], s, 128), vh[t, h], atol=1e-12)


def test_attention_bruteforce():
    """reference_attention semantics: q_to_req / q_to_klen through the block
    table, GQA by repeat_interleave, zero rows for klen <= 0."""
    s = synth.sign_pattern(128)
    nreq, Hkv, Hq, bs, nblk = 2, 2, 4, 16, 8
    k = synth.gaussian(11, (nblk * bs, Hkv, 128))
    v = synth.gaussian(12, (nblk * bs, Hkv, 128))
    slots = oracle.octave_quantize(k, v, FMT, s)                      # (T, H, slot)
    cache = slots.reshape(nblk, bs, Hkv, 128).transpose(0, 2, 1, 3).copy()  # (blocks, Hkv, bs, slot)
    bt = np.array([[5, 2, 7, 0], [1, 3, 4, 6]], np.int32)
    q = synth.gaussian(13, (4, Hq, 128))
    q_to_req = np.array([0, 1, 1, 0], np.int32)
    q_to_klen = np.array([50, 64, 0, 7], np.int32)
    got = oracle.octave_attention(q, cache, bt, q_to_req, q_to_klen, FMT, 0.09, s)
    kd, vd = oracle.octave_dequantize(cache.transpose(0, 2, 1, 3).reshape(-1, Hkv, 128), FMT, s)
    kd = kd.reshape(nblk, bs, Hkv, 128)
    vd = vd.reshape(nblk, bs, Hkv, 128)
    for i in range(4):
        L = q_to_klen[i]
        if L <= 0:
            assert np.all(got[i] == 0)
            continue
        pos = np.arange(L)
        blk = bt[q_to_req[i], pos // bs]
        K = kd[blk, pos % bs]
        V = vd[blk, pos % bs]
        for h in range(Hq):
            g = h // (Hq // Hkv)
            sc = 0.09 * (K[:, g] @ q[i, h].astype(np.float64))
            p = np.exp(sc - sc.max())
            p /= p.sum()
            np.testing.assert_allclose(got[i, h], p @ V[:, g], atol=1e-12)


# ---------------------------------------------------------------------------
# Hand-derived goldens for _quantize_lut and for the slot assembly of
# reference_quantize, and planted misreadings that each of them catches.
# ---------------------------------------------------------------------------
LUT_GOLD = json.load(open(os.path.join(GOLD, "octave_quantize_lut.json")))
SLOT_GOLD = json.load(open(os.path.join(GOLD, "octave_slot_k3v4.json")))


def _bits32(v):
    return "0x%08x" % int(np.float32(v).view(np.uint32))


def test_lut_golden_inputs_are_the_codebook():
    for bits in (3, 4):
        lut, mult = oracle.octave_codebook(bits)
        assert lut.tolist() == LUT_GOLD["inputs"][f"lut{bits}"]
        assert _bits32(mult) == LUT_GOLD["inputs"][f"lut_mult{bits}_bits"]


def _check_lut_case(qlut, f16, case):
    x = np.array([np.uint32(int(b, 16)).view(np.float32) for b in case["x_bits"]], np.float32)
    codes, scale = qlut(x, case["bits"])
    assert list(codes) == case["codes"], "codes"
    assert _bits32(scale) == case["scale_f32_bits"], "fp32 scale"
    assert "0x%04x" % f16(scale) == case["scale_f16_bits"], "fp16 scale"


@pytest.mark.parametrize("case", LUT_GOLD["cases"], ids=lambda c: c["name"])
def test_quantize_lut_golden(case):
    _check_lut_case(oracle.octave_quantize_lut,
                    lambda s: int(oracle.f32_to_f16_bits(np.array([s], np.float32))[0]), case)


def _slot_inputs():
    s = np.ones(128, np.float32)
    s[[1, 70, 127]] = -1
    walsh = lambda i, k: -1.0 if bin(i & k).count("1") % 2 else 1.0
    k = np.zeros((1, 1, 128), np.float32)
    v = np.zeros((1, 1, 128), np.float32)
    for i in range(64):
        k[0, 0, i] = s[i] * np.float32(3 / 8) * walsh(i, 5)
        k[0, 0, 64 + i] = s[64 + i] * np.float32(-5 / 8) * walsh(i, 9)
    for i in range(128):
        v[0, 0, i] = s[i] * np.float32(0.5) * walsh(i, 100)
    return k, v, s


def test_slot_golden_k3v4():
    k, v, s = _slot_inputs()
    slot = oracle.octave_quantize(k, v, tuple(SLOT_GOLD["format"]), s)[0, 0]
    assert slot.tobytes().hex() == SLOT_GOLD["slot_hex"]


# Each entry plants one plausible misreading in a copy of the oracle source
# (the oracle itself is untouched); at least one golden must then fail.
PLANTED = {
    "bucketize right=True": ("if (mid[k] < y) c++;", "if (mid[k] <= y) c++;"),
    "ss summed left to right": ("float ss = tree_sum_f32(tmp, n);",
                                "float ss = 0.0f; for (int i = 0; i < n; i++) ss = ss + tmp[i];"),
    "dot summed left to right": ("float dot = tree_sum_f32(tmp, n);",
                                 "float dot = 0.0f; for (int i = 0; i < n; i++) dot = dot + tmp[i];"),
    "y with one rounding": ("float y = x[i] / rms;\n    y = y * mult;", "float y = x[i] * (mult / rms);"),
    "fp16 half up": ("if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h++;",
                     "if (rem >= 0x1000u) h++;"),
    "V scale before K scales": ("uint16_t hb = orc_f32_to_f16(scales[s]);",
                                "uint16_t hb = orc_f32_to_f16(scales[(s + f.num_k_scales) % f.num_scales]);"),
    "pad bytes not zero": ("memset(slot, 0, (size_t)f.slot_bytes);",
                           "memset(slot, 0x5a, (size_t)f.slot_bytes);"),
    "sign flips skipped": ("for (int i = 0; i < d; i++) x[i] = x[i] * signs[i];", ""),
    "RoPE and NoPE bit widths swapped": (
        "int bits = kb < f.num_rope_blocks ? OCT_ROPE_BITS : OCT_NOPE_BITS;",
        "int bits = kb < f.num_rope_blocks ? OCT_NOPE_BITS : OCT_ROPE_BITS;"),
}


def _planted_lib(tmp_path, old, new):
    import ctypes as C
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kvq_oracle.c")).read()
    assert src.count(old) == 1, f"pattern not found once in the oracle: {old!r}"
    path = tmp_path / "planted.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "planted.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-I", os.path.dirname(oracle.__file__),
                           "-o", str(so), str(path), "-lm"])
    L = C.CDLL(str(so))
    L.orc_f32_to_f16.restype = C.c_uint16
    L.orc_f32_to_f16.argtypes = [C.c_float]
    return L


def _goldens_pass(L):
    import ctypes as C

    def qlut(x, bits):
        codes = np.zeros(x.size, np.uint8)
        s = C.c_float(0)
        r = L.orc_octave_quantize_lut(x.ctypes.data_as(C.c_void_p), x.size, bits,
                                      codes.ctypes.data_as(C.c_void_p), C.byref(s))
        assert r == 0
        return codes, np.float32(s.value)

    ok = True
    for case in LUT_GOLD["cases"]:
        try:
            _check_lut_case(qlut, lambda s: int(L.orc_f32_to_f16(float(s))), case)
        except AssertionError:
            ok = False
    k, v, s = _slot_inputs()
    out = np.zeros(128, np.uint8)
    r = L.orc_octave_quantize(128, 64, 4, 0, k.ctypes.data_as(C.c_void_p),
                              v.ctypes.data_as(C.c_void_p), 0, 1, 1,
                              s.ctypes.data_as(C.c_void_p), out.ctypes.data_as(C.c_void_p))
    assert r == 0
    return ok and out.tobytes().hex() == SLOT_GOLD["slot_hex"]


def test_goldens_pass_on_unplanted_copy(tmp_path):
    assert _goldens_pass(_planted_lib(tmp_path, "#define OCT_HB 64", "#define OCT_HB 64"))


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_goldens_catch_planted_misreading(tmp_path, name):
    old, new = PLANTED[name]
    assert not _goldens_pass(_planted_lib(tmp_path, old, new)), f"{name} went unnoticed"
