"""Dense -> g128 quantiser on the GPU against the oracle's least-squares fit: the codes, the fp16
scales and the packed words / bytes are bit-exact, for the three storages and the three input
types, on random weights and on groups chosen to stress the selection (zeros, a single non-zero,
equal magnitudes, magnitudes spread over many binades)."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import bq, requires_gpu

pytestmark = requires_gpu

FMTS = [(oracle.BINARY, 0), (oracle.TERNARY, 1), (oracle.TERNARY_B3, 2)]


def dense(seed, N, K):
    return (synth.activations(seed, N, K, dtype=torch.float32) * 0.02).float()


def check(orc, w, ofmt, dfmt):
    m = bq()
    pw = m.quantize_g128(w.cuda(), dfmt)
    torch.cuda.synchronize()
    w32 = w.float().numpy()
    q_ref, s_ref = orc.quantize(ofmt if ofmt != oracle.TERNARY_B3 else oracle.TERNARY, w32)
    s_dev = pw.scales.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(s_dev, s_ref), f"scales differ in {np.sum(s_dev != s_ref)} groups"
    st, packed_ref, _ = orc.pack(ofmt, q_ref, s_ref.view(np.float16))
    assert st == oracle.OK
    got = pw.words.cpu().numpy()
    if ofmt != oracle.TERNARY_B3:
        got = got.view(np.uint32)
    assert np.array_equal(got, packed_ref)
    q_dev, _ = m.unpack_g128(pw)
    assert np.array_equal(q_dev.cpu().numpy(), q_ref)


@pytest.mark.parametrize("wdt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("ofmt,dfmt", FMTS)
def test_quantize_random(orc, ofmt, dfmt, wdt):
    w = dense(11, 300, 1152).to(wdt)
    check(orc, w, ofmt, dfmt)


@pytest.mark.parametrize("ofmt,dfmt", FMTS)
def test_quantize_special_groups(orc, ofmt, dfmt):
    K = 1024
    w = dense(12, 8, K)
    w[0, :128] = 0.0                                  # a group of zeros
    w[1, :128] = 0.0
    w[1, 77] = -0.5                                   # a single non-zero
    w[2, :128] = 0.25 * torch.tensor([(-1) ** k for k in range(128)])   # equal magnitudes
    w[3, :128] = torch.tensor([2.0 ** (-(k % 25)) for k in range(128)])  # 25 binades
    w[4, :64] = 1.0
    w[4, 64:128] = 0.001                              # two clusters
    w[5, 128:256] = torch.linspace(-1, 1, 128)
    w[6, :128] = 0.0
    w[6, :4] = torch.tensor([3.0, -1.0, 1.0, -1.0])     # equal scores at j = 1 and j = 4: j = 1
    check(orc, w, ofmt, dfmt)


@pytest.mark.parametrize("ofmt,dfmt", FMTS)
def test_quantize_k5120_n5120(orc, ofmt, dfmt):
    check(orc, dense(13, 5120, 5120).to(torch.bfloat16), ofmt, dfmt)


def test_quantize_ternary_beats_absmean(orc):
    """The least-squares ternary fit has no larger squared error than the common absmean rule
    (s = mean |w|, q = round(clip(w / s, -1, 1))) on any group."""
    m = bq()
    N, K = 64, 1024
    w = dense(14, N, K)
    pw = m.quantize_g128(w.cuda(), m.TERNARY_G128)
    q, s = m.unpack_g128(pw)
    wg = w.double().view(N, K // 128, 128)
    fit = q.cpu().double().view(N, K // 128, 128) * s.cpu().double().unsqueeze(-1)
    err_ls = ((wg - fit) ** 2).sum(-1)
    gam = wg.abs().mean(-1, keepdim=True)
    qa = torch.clamp(torch.round(wg / gam), -1, 1)
    err_am = ((wg - qa * gam.half().double()) ** 2).sum(-1)
    assert torch.all(err_ls <= err_am * (1 + 1e-3) + 1e-12)


def test_quantize_errors():
    m = bq()
    w = torch.zeros((4, 200), device="cuda")
    with pytest.raises(m.BQError) as e:
        m.quantize_g128(w, m.BINARY_G128)
    assert e.value.status_name == "BQ_ERR_SHAPE"
