"""GPU parity of multi-token decode (kvq_decode_attn_multi): several query
tokens per sequence, each over its own causal prefix, against the oracle's
attention of that sequence prefix; a query whose sequence index is outside
the cache gets a zero row."""
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


def to_dev(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def oracle_rows(oc, q, q_to_seq, q_lens, n_seqs, scale):
    """Query i through the oracle: a batch with q[i] in the row of its sequence."""
    want = np.zeros(q.shape, np.float64)
    for i in range(len(q)):
        s = int(q_to_seq[i])
        if s < 0 or s >= n_seqs:
            continue
        qb = np.zeros((n_seqs,) + q.shape[1:], q.dtype)
        qb[s] = q[i]
        lens = np.zeros(n_seqs, np.int32)
        lens[s] = q_lens[i]
        want[i] = oc.decode_attn(qb, lens, scale)[s]
    return want


@pytest.mark.parametrize("G", [4, 8])
def test_multi_contiguous(G):
    B, H, T = 3, 2, 800
    k, v = synth.kv_tokens(510 + G, B, T, H, 256, 0.01, 16.0)
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.contiguous(B, H, T)
    kvq.quantize_append(gc, to_dev(k), to_dev(v), to_dev(np.zeros(B, np.int32)))
    oc = oracle.Q4Cache(B * H * T, H, max_tokens=T)
    oc.append(k, v, np.zeros(B, np.int32))
    # three drafted tokens of sequence 0, one query each of sequences 1 and 2,
    # a second one of sequence 2, and one with no sequence
    q_to_seq = np.array([0, 0, 0, 1, 2, 2, 5], np.int32)
    q_lens = np.array([798, 799, 800, 300, 1, 64, 100], np.int32)
    q = synth.to_bf16_bits(synth.queries(520 + G, len(q_to_seq), H * G, 256))
    got = kvq.decode_attn_multi(gc, to_dev(q), to_dev(q_to_seq), to_dev(q_lens), B, T,
                                1 / 16).cpu().numpy()
    want = oracle_rows(oc, q, q_to_seq, q_lens, B, 1 / 16)
    assert np.abs(got - want).max() <= ATOL
    assert not np.any(got[6])


def test_multi_paged():
    B, H, G, ps = 2, 2, 8, 64
    lens = np.array([500, 190], np.int32)
    T = int(lens.max())
    npp = np.array([(int(L) + ps - 1) // ps for L in lens])
    bt, n_pages = synth.page_table(31, B, npp, int(npp.max()) + 1, extra_pages=3)
    k, v = synth.kv_tokens(530, B, T, H, 256, 0.01, 16.0)
    k, v = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    gc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt))
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    for b in range(B):
        L = int(lens[b])
        sp = np.zeros(1, np.int32)
        kvq.quantize_append(gc.with_block_table(torch.from_numpy(bt[b:b + 1])),
                            to_dev(k[b:b + 1, :L]), to_dev(v[b:b + 1, :L]), to_dev(sp))
        oc.with_block_table(bt[b:b + 1]).append(k[b:b + 1, :L], v[b:b + 1, :L], sp)
    q_to_seq = np.array([1, 0, 0, 0, 0, 1], np.int32)
    q_lens = np.array([190, 497, 498, 499, 500, 129], np.int32)
    q = synth.queries(540, len(q_to_seq), H * G, 256)  # fp32 queries
    got = kvq.decode_attn_multi(gc, to_dev(q), to_dev(q_to_seq), to_dev(q_lens), B, T,
                                1 / 16).cpu().numpy()
    want = oracle_rows(oc, q, q_to_seq, q_lens, B, 1 / 16)
    assert np.abs(got - want).max() <= ATOL
