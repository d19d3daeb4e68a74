"""GPU pack / unpack against the oracle: bit-exact words, validation of the value set."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import bq, requires_gpu

pytestmark = requires_gpu


@pytest.mark.parametrize("N,K", [(1, 128), (3, 640), (300, 1152), (1000, 5120)])
def test_pack_binary_bit_exact(orc, N, K):
    m = bq()
    q = synth.random_signs(20 + N, synth.TID_SIGNS, (N, K))
    s = synth.scales(20 + N, N, K // 128)
    w = m.pack_binary_g128(q.cuda(), s.cuda())
    st, words_ref, s_ref = orc.pack(oracle.BINARY, q.numpy(), s.numpy())
    assert st == oracle.OK
    assert np.array_equal(w.words.cpu().numpy().view(np.uint32), words_ref)
    assert np.array_equal(w.scales.cpu().numpy().view(np.uint16), s_ref)
    q2, s2 = m.unpack_g128(w)
    assert torch.equal(q2.cpu(), q) and torch.equal(s2.cpu(), s)


@pytest.mark.parametrize("N,K", [(1, 128), (5, 384), (777, 2048), (2048, 5120)])
def test_pack_ternary_bit_exact(orc, N, K):
    m = bq()
    q = synth.random_ternary(30 + N, synth.TID_TERNARY, (N, K))
    s = synth.scales(30 + N, N, K // 128)
    w = m.pack_ternary_g128(q.cuda(), s.cuda())
    st, words_ref, _ = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
    assert st == oracle.OK
    assert np.array_equal(w.words.cpu().numpy().view(np.uint32), words_ref)
    q2, _ = m.unpack_g128(w)
    assert torch.equal(q2.cpu(), q)


def test_unpack_of_random_words_matches_oracle(orc):
    m = bq()
    N, K = 64, 1024
    words = synth.binary_words(40, N, K)
    s = synth.scales(40, N, K // 128)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    q, _ = m.unpack_g128(w)
    q_ref, bad = orc.unpack(oracle.BINARY, words.numpy(), K)
    assert bad == 0 and np.array_equal(q.cpu().numpy(), q_ref)
    # and packing it again reproduces the words
    w2 = m.pack_binary_g128(q, w.scales)
    assert torch.equal(w2.words, w.words)


def test_pack_rejects_values_outside_the_set():
    m = bq()
    K = 256
    q = torch.ones((4, K), dtype=torch.int8)
    q[2, 100] = 0
    s = torch.ones((4, 2), dtype=torch.float16)
    with pytest.raises(m.BQError) as e:
        m.pack_binary_g128(q.cuda(), s.cuda())
    assert e.value.status_name == "BQ_ERR_INVALID_CODE"
    qt = torch.zeros((4, K), dtype=torch.int8)
    qt[3, 7] = 2
    with pytest.raises(m.BQError) as e:
        m.pack_ternary_g128(qt.cuda(), s.cuda())
    assert e.value.status_name == "BQ_ERR_INVALID_CODE"
    # a valid call afterwards succeeds (the counter was reset)
    m.pack_binary_g128(torch.ones((4, K), dtype=torch.int8).cuda(), s.cuda())


def test_unpack_reports_ternary_code3(orc):
    m = bq()
    N, K = 2, 128
    words = torch.zeros((N, K // 16), dtype=torch.int32)
    words[1, 3] = 0x3 << 10                                   # k = 53 of row 1
    w = m.BQWeight(m.TERNARY_G128, N, K, words.cuda(), torch.ones((N, 1), dtype=torch.float16).cuda())
    with pytest.raises(m.BQError) as e:
        m.unpack_g128(w)
    assert e.value.status_name == "BQ_ERR_INVALID_CODE"
    q_ref, bad = orc.unpack(oracle.TERNARY, words.numpy(), K)
    assert bad == 1 and q_ref[1, 53] == 0
