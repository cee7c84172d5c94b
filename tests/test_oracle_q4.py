"""Pins for the oracle's Q4_0 quantizer (Strata PR #21: How 2 and the
maintainer's deterministic-quantization note; GGML Q4_0 reading)."""
import json
import os

import numpy as np
import pytest

import oracle
from hadamard_rotated_bit_fwht_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _block(spec):
    z = np.zeros(32, np.float32)
    for k, v in spec.items():
        z[int(k)] = v
    return z


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLD, "q4_0_blocks.json")))["cases"],
                         ids=lambda c: c["name"])
def test_hand_built_blocks(case):
    qs, d = oracle.q4_0_block(_block(case["z"]))
    assert qs.tobytes().hex() == case["qs_hex"]
    assert d == int(case["d_bits"], 16)


def test_tie_dequant_values():
    # [+1, -1, 0...]: codes 0 and 15 with d = -0.125 -> +1.0 and -0.875 (clamped)
    qs, d = oracle.q4_0_block(_block({"0": 1.0, "1": -1.0}))
    deq = oracle.q4_0_dequant_block(qs, d)
    assert deq[0] == 1.0 and deq[1] == -0.875 and np.all(deq[2:] == 0.0)


def _lexmax(z):
    """The tie-break rule restated as a maximum: the element with the largest
    |z|, the positive one among equal magnitudes; start value (0, +0)."""
    best = (0.0, 0.0)
    for v in z.tolist():
        best = max(best, (abs(v), v))
    return np.float32(best[1])


def test_scale_is_order_independent_lexmax():
    rng = np.random.default_rng(7)
    for trial in range(300):
        z = rng.standard_normal(32).astype(np.float32)
        if trial % 3 == 0:  # force exact magnitude ties of both signs
            z[rng.integers(32)] = -np.abs(z).max()
            z[rng.integers(32)] = np.abs(z).max()
        qs, d = oracle.q4_0_block(z)
        mval = _lexmax(z)
        assert d == int((mval / np.float32(-8.0)).astype(np.float16).view(np.uint16))
        perm = rng.permutation(32)
        qs2, d2 = oracle.q4_0_block(z[perm])
        assert d2 == d
        codes = np.concatenate([qs & 15, qs >> 4])
        codes2 = np.concatenate([qs2 & 15, qs2 >> 4])
        np.testing.assert_array_equal(codes2, codes[perm])


def test_error_bound():
    """|z - z_hat| <= amax/16 (+ fp16 scale rounding) for every element, except
    elements of the sign opposite to mval with |z| > 15/16 amax, which clamp to
    code 15 and are bounded by amax/8."""
    rng = np.random.default_rng(3)
    z = rng.standard_normal((4000, 32)).astype(np.float32) * rng.uniform(1e-3, 50, (4000, 1)).astype(np.float32)
    z[::7, 3] *= 16  # outliers
    for row in z:
        qs, d = oracle.q4_0_block(row)
        deq = oracle.q4_0_dequant_block(qs, d)
        amax = np.abs(row).max()
        mval = _lexmax(row)
        err = np.abs(row.astype(np.float64) - deq)
        slack = 8 * max(amax / 8 * 2.0 ** -11, 2.0 ** -25) + amax * 2.0 ** -20
        clamp = (np.sign(row) == -np.sign(mval)) & (np.abs(row) > amax * 15 / 16)
        assert np.all(err[~clamp] <= amax / 16 + slack)
        assert np.all(err[clamp] <= amax / 8 + slack)


def test_fwht_lowers_int4_error_on_outlier_channels():
    """The qualitative claim (Strata PR #21 Why; Round 40 audit item #5): a
    Hadamard rotation before 4-bit block quantization lowers the error on data
    with outlier channels.  Informational bound, not a value from the pages."""
    k, _ = synth.kv_tokens(seed=2, batch=1, n_tok=512, n_kv_heads=2, dim=256,
                           outlier_frac=0.01, outlier_factor=16.0)
    x = k.reshape(-1, 256)
    # with rotation: oracle quantizes H x; dequantize and rotate back
    codes, scales = oracle.q4_quantize_vectors(x)
    deq = np.stack([np.concatenate([oracle.q4_0_dequant_block(codes[i, b * 16:(b + 1) * 16],
                                                              scales[i, b]) for b in range(8)])
                    for i in range(x.shape[0])])
    rec = oracle.fwht_f64(deq)
    err_rot = np.linalg.norm(rec - x) / np.linalg.norm(x)
    # without rotation: quantize x directly block by block
    deq2 = []
    for row in x:
        parts = []
        for b in range(8):
            qs, d = oracle.q4_0_block(row[b * 32:(b + 1) * 32])
            parts.append(oracle.q4_0_dequant_block(qs, d))
        deq2.append(np.concatenate(parts))
    err_raw = np.linalg.norm(np.stack(deq2) - x) / np.linalg.norm(x)
    assert err_rot < err_raw


def test_vectors_equal_rotate_then_blocks():
    """q4_quantize_vectors is FWHT-256 (fp32) followed by eight Q4_0 blocks."""
    rng = np.random.default_rng(9)
    x32 = rng.standard_normal((20, 256)).astype(np.float32)
    xb = synth.to_bf16_bits(x32)
    codes, scales = oracle.q4_quantize_vectors(xb)
    y = oracle.fwht_f32(synth.bf16_bits_to_f32(xb))
    for i in range(20):
        for b in range(8):
            qs, d = oracle.q4_0_block(y[i, b * 32:(b + 1) * 32])
            assert codes[i, b * 16:(b + 1) * 16].tobytes() == qs.tobytes() and scales[i, b] == d


def test_append_layouts_agree():
    """Contiguous and paged appends store identical bytes per (b, h, t)."""
    B, H, T = 2, 3, 40
    k = synth.to_bf16_bits(synth.gaussian(100, (B, T, H, 256)))
    v = synth.to_bf16_bits(synth.gaussian(101, (B, T, H, 256)))
    cc = oracle.Q4Cache(B * H * 64, H, max_tokens=64)
    cc.append(k[:, :25], v[:, :25], [0, 0])
    cc.append(k[:, 25:], v[:, 25:], [25, 25])
    ps = 16
    bt, n_pages = synth.page_table(4, B, np.array([3, 3]), 4, extra_pages=2)
    pc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    pc.append(k, v, [0, 0])
    for b in range(B):
        for h in range(H):
            for t in range(T):
                rc = (b * H + h) * 64 + t
                rp = (bt[b, t // ps] * H + h) * ps + t % ps
                assert cc.k_codes[rc].tobytes() == pc.k_codes[rp].tobytes()
                assert cc.v_scales[rc].tobytes() == pc.v_scales[rp].tobytes()
