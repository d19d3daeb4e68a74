"""GPU embedding gather against the oracle: bit-exact after the same rounding."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import bq, requires_gpu

pytestmark = requires_gpu


def _ref16(orc, out_ref, dt):
    if dt == torch.bfloat16:
        return orc.to_bf16_bits(out_ref)
    return out_ref.astype(np.float16).view(np.uint16)         # fp16 +-s is exact


@pytest.mark.parametrize("ot", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_embed_small(orc, fmt, ot):
    m = bq()
    N, K, T = 1000, 640, 77
    s = synth.scales(50, N, K // 128)
    if fmt == 0:
        words = synth.binary_words(50, N, K)
        w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
        wref = words.numpy()
    else:
        q = synth.random_ternary(50, synth.TID_TERNARY, (N, K))
        w = m.pack_ternary_g128(q.cuda(), s.cuda())
        _, wref, _ = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
    ids = synth.random_ids(50, synth.TID_IDS, T, N)
    out = m.embed_gather(ids.cuda(), w, out_dtype=ot).cpu()
    ref, bad = orc.embed(fmt, ids.numpy(), wref, s, K)
    assert bad == 0
    if ot == torch.float32:
        assert np.array_equal(out.numpy().astype(np.float64), ref)
    else:
        got = out.view(torch.int16).numpy().view(np.uint16)
        exp = _ref16(orc, ref, ot)
        # compare values so that +0 / -0 of a zero scale count as equal
        gv = torch.from_numpy(got.view(np.int16)).view(ot).float()
        ev = torch.from_numpy(exp.view(np.int16)).view(ot).float()
        assert torch.equal(gv, ev)


def test_embed_vocab_4096_ids(orc):
    """4096 ids uniform in [0, 248320) over the K=5120 binary matrix, bf16 output."""
    m = bq()
    N, K, T = 248320, 5120, 4096
    words = synth.binary_words(0, N, K)
    s = synth.scales(0, N, K // 128)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    ids = synth.random_ids(0, synth.TID_IDS, T, N)
    out = m.embed_gather(ids.cuda(), w).cpu()
    m.get_device_error()
    ref, bad = orc.embed(0, ids.numpy(), words, s, K)
    assert bad == 0
    assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), orc.to_bf16_bits(ref))


def test_embed_out_of_range_ids(orc):
    m = bq()
    N, K = 100, 256
    words = synth.binary_words(60, N, K)
    s = synth.scales(60, N, K // 128)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    ids = torch.tensor([5, -1, 100, 99], dtype=torch.int32)
    m.get_device_error()                                       # clear anything earlier
    out = m.embed_gather(ids.cuda(), w, out_dtype=torch.float32).cpu()
    with pytest.raises(m.BQError) as e:
        m.get_device_error()
    assert e.value.status_name == "BQ_ERR_INVALID_ARG"
    m.get_device_error()                                       # cleared by the read
    ref, bad = orc.embed(0, ids.numpy(), words, s, K)
    assert bad == 2
    assert np.array_equal(out.numpy().astype(np.float64), ref)
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)


def test_embed_empty():
    m = bq()
    N, K = 10, 128
    w = m.BQWeight(m.BINARY_G128, N, K, synth.binary_words(1, N, K).cuda(),
                   synth.scales(1, N, 1).cuda())
    out = m.embed_gather(torch.empty(0, dtype=torch.int32, device="cuda"), w)
    assert out.shape == (0, K)
