"""The adversarial prefill inputs really are adversarial (CPU only): with each fp16 scale
rounded to bf16 (torch's round-to-nearest-even conversion), the product breaks the
2e-3 * sum|x s| bound that the oracle computes, by about 2x. So the GPU tests that feed these
inputs would catch a bf16-rounded +-s operand."""

import numpy as np
import torch

import oracle
from tests.adversarial import (TIE_SCALES, adversarial_binary, adversarial_ternary_q,
                               positive_bf16_x)


def test_tie_scales_are_bf16_ties(orc):
    for b in TIE_SCALES:
        s = orc.f16_value(b)
        r = float(torch.tensor([s], dtype=torch.float64).to(torch.bfloat16).double())
        assert abs(r - s) / s > 2.5e-3, hex(b)          # more than the relative tolerance


def _y_with_bf16_scales(orc, fmt, words, s, K, x):
    s_bf = s.to(torch.bfloat16).to(torch.float64).numpy()
    W = orc.dequant(fmt, words, np.ones(s.shape, dtype=np.float16), K)   # +-1 / 0 per weight
    Wb = W * np.repeat(s_bf, 128, axis=1)
    return x.to(torch.float64).numpy() @ Wb.T


def test_binary_fixture_breaks_bf16_scales(orc):
    N, K, M = 64, 512, 3
    words, s = adversarial_binary(N, K)
    x = positive_bf16_x(1, M, K)
    y_ref, bound = orc.gemv(oracle.BINARY, x, oracle.X_BF16, words, s, K)
    y_bad = _y_with_bf16_scales(orc, oracle.BINARY, words, s, K, x)
    ratio = np.max(np.abs(y_bad - y_ref) / bound)
    assert ratio > 1.5, ratio


def test_ternary_fixture_breaks_bf16_scales(orc):
    N, K, M = 64, 512, 3
    q, s = adversarial_ternary_q(N, K)
    st, words, _ = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
    assert st == oracle.OK
    x = positive_bf16_x(2, M, K)
    y_ref, bound = orc.gemv(oracle.TERNARY, x, oracle.X_BF16, words, s, K)
    y_bad = _y_with_bf16_scales(orc, oracle.TERNARY, words, s, K, x)
    ratio = np.max(np.abs(y_bad - y_ref) / bound)
    assert ratio > 1.5, ratio
