"""The bounds-checking build (libkvq_debug.so, compiled with KVQ_DEBUG_BOUNDS):
every computed cache row, scale-row run and Octave slot is checked against the
buffer the call describes, and a violation is recorded in the device error
word instead of being accessed.  Run in a child process that loads that build
(KVQ_LIBRARY), over Q4_0 / Q8_0 appends and decodes (contiguous, paged with an
unmapped page, fused step, several queries per sequence, the allocation-free
call) and the Octave quantize and decode: the results match the oracle as the
release build's do, and the error word stays clean."""
import os
import subprocess
import sys
import textwrap

import pytest

from hadamard_rotated_bit_fwht_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import numpy as np, torch
    import oracle
    from hadamard_rotated_bit_fwht_b200 import kvq, synth
    assert kvq.LIB_PATH.endswith("libkvq_debug.so"), kvq.LIB_PATH
    dev = lambda a: (torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16)
                     if a.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(a))).cuda()
    worst = 0.0
    for bits in (4, 8):
        B, H, G, T = 2, 2, 8, 700
        k, v = synth.kv_tokens(41 + bits, B, T, H, 256, 0.01, 16.0)
        kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
        q = synth.to_bf16_bits(synth.queries(42, B, H * G, 256))
        gc = kvq.Q4Cache.contiguous(B, H, T, bits=bits)
        kvq.quantize_append(gc, dev(kb[:, :T - 1]), dev(vb[:, :T - 1]), dev(np.zeros(B, np.int32)))
        out = kvq.decode_step(gc, dev(kb[:, T - 1]), dev(vb[:, T - 1]), dev(q),
                              dev(np.full(B, T - 1, np.int32)), T, 1 / 16)
        oc = oracle.Q4Cache(B * H * T, H, max_tokens=T, bits=bits)
        oc.append(kb, vb, np.zeros(B, np.int32))
        worst = max(worst, np.abs(out.cpu().numpy() - oc.decode_attn(q, [T, T], 1 / 16)).max())
        kvq.decode_attn_multi(gc, dev(q[[0, 1, 0]]), dev(np.array([0, 1, 0], np.int32)),
                              dev(np.array([T, 300, 17], np.int32)), B, T, 1 / 16)
        # paged, one page of sequence 1 unmapped (it contributes nothing)
        ps = 64
        npp = np.array([11, 11])
        bt, n_pages = synth.page_table(43, B, npp, 12, extra_pages=1)
        pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), bits=bits)
        kvq.quantize_append(pc, dev(kb), dev(vb), dev(np.zeros(B, np.int32)))
        bt2 = bt.copy(); bt2[1, 3] = -1
        kvq.decode_attn(pc.with_block_table(torch.from_numpy(bt2)), dev(q),
                        dev(np.array([T, T], np.int32)), T, 1 / 16)
        kvq.decode_attn_noalloc(gc, dev(q), dev(np.array([T, 5], np.int32)), T, 1 / 16)
    F = kvq.OctaveFormat(128, 64, 4)
    fmt = (128, 64, 4, 0)
    Tn, Hkv, bs = 300, 2, 16
    k = synth.to_bf16_bits(synth.gaussian(44, (Tn, Hkv, 128)))
    v = synth.to_bf16_bits(synth.gaussian(45, (Tn, Hkv, 128)))
    nblk = (Tn + bs - 1) // bs
    slot = np.arange(Tn, dtype=np.int64)
    signs = synth.sign_pattern(128)
    cache = torch.zeros((nblk, Hkv, bs, 128), dtype=torch.uint8, device="cuda")
    kvq.octave_quantize(F, dev(k), dev(v), dev(slot), cache, kvq.sign_words(signs))
    want = oracle.octave_quantize(k, v, fmt, signs)
    got = cache.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, Hkv, 128)[:Tn]
    assert np.array_equal(got, want), "octave slots"
    bt = np.arange(nblk, dtype=np.int32)[None]
    qo = synth.to_bf16_bits(synth.gaussian(46, (1, 8, 128)))
    o = kvq.octave_decode_attn(F, dev(qo), cache, dev(bt), dev(np.zeros(1, np.int32)),
                               dev(np.array([Tn], np.int32)), Tn, 128 ** -0.5,
                               kvq.sign_words(signs)).cpu().numpy()
    wo = oracle.octave_attention(qo, cache.cpu().numpy(), bt, np.zeros(1, np.int32),
                                 np.array([Tn], np.int32), fmt, 128 ** -0.5, signs)
    worst = max(worst, np.abs(o - wo).max())
    torch.cuda.synchronize()
    print("worst", worst, "flags", kvq.device_errors())
""")


def test_debug_build_is_clean_and_exact():
    lib = build.build(debug=True)
    env = dict(os.environ, KVQ_LIBRARY=lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    last = r.stdout.strip().splitlines()[-1].split()
    assert float(last[1]) <= 2e-3, r.stdout
    assert int(last[3]) == 0, f"bounds violations recorded: {r.stdout}"
