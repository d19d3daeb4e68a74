"""bq_gemv_noalloc (the decode GEMV with the library's fixed scratch array) against bq_gemv
with a caller workspace, through the C ABI. Two calls in a row per shape, each within the
GEMV tolerance max|y - y_ws| <= 2e-3 * sum_k |x s| of the workspace call's result (the same
kernel and the same fixed summation order, so the outputs are also bit-identical). On these
shapes the prep kernel writes the digit fragments of x into the array and the GEMV reads them
back from it. Collected last, so it also runs after every other test has used the library."""

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_common import binary_inputs, bq, requires_gpu, sample_rows, ternary_q

pytestmark = requires_gpu


def _weights(m, fmt, seed, N, K, M, orc=None):
    x, words, s = binary_inputs(seed, N, K, M)
    if fmt == m.BINARY_G128:
        return x, m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda()), words, s
    st, words, s_ref = orc.pack(oracle.TERNARY, ternary_q(seed, N, K).numpy(), s.numpy())
    assert st == oracle.OK
    wd = torch.from_numpy(words.view(np.int32)).cuda()
    sd = torch.from_numpy(s_ref.view(np.float16)).cuda()
    return x, m.BQWeight(m.TERNARY_G128, N, K, wd, sd), words, s_ref


def _bound(orc, fmt, x, words, s, K, rows):
    code = oracle.BINARY if fmt == 0 else oracle.TERNARY
    _, bound = orc.gemv(code, x, oracle.X_BF16, words, s, K, rows=rows)
    return bound


@pytest.mark.parametrize("fmt,N,K,M", [
    (0, 20480, 5120, 8),      # four column sets: the largest fragment set at K = 5120
    (0, 248320, 5120, 1),     # the LM head
    (1, 20480, 5120, 4),      # ternary
    (0, 1000, 640, 3),        # K not a multiple of 1024: the kernel that needs no scratch
])
def test_noalloc_matches_workspace_call(orc, fmt, N, K, M):
    m = bq()
    x, w, words, s = _weights(m, fmt, 31 + M, N, K, M, orc)
    xd = x.cuda()
    ws = torch.empty(max(m.gemv_workspace_bytes(M, w), 1), dtype=torch.uint8, device="cuda")
    y_ws = m.gemv(xd, w, workspace=ws)
    rows = sample_rows(N, 600, M)
    bound = _bound(orc, fmt, x, words, s, K, rows)
    ref = y_ws[:, torch.from_numpy(rows).cuda()].double().cpu().numpy()
    for call in range(2):
        y = m.gemv_noalloc(xd, w)
        torch.cuda.synchronize()
        got = y[:, torch.from_numpy(rows).cuda()].double().cpu().numpy()
        err = np.abs(got - ref)
        assert np.all(err <= bound), f"call {call}: max err/bound = {np.max(err / bound):.3g}"
        assert torch.equal(y, y_ws), f"call {call}: differs from the workspace call"
    m.get_device_error()                  # raises if a bounded wait gave up


def test_noalloc_allocates_nothing():
    """After a first call (which resolves the array once), repeated calls leave the device's
    free memory unchanged."""
    m = bq()
    N, K, M = 20480, 5120, 8
    x, w, _, _ = _weights(m, 0, 5, N, K, M)
    xd = x.cuda()
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    m.gemv_noalloc(xd, w, out=y)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        m.gemv_noalloc(xd, w, out=y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_bad_arguments():
    m = bq()
    x, w, _, _ = _weights(m, 0, 9, 256, 1024, 1)
    with pytest.raises(m.BQError) as e:
        m.gemv_noalloc(torch.zeros((9, 1024), dtype=torch.bfloat16, device="cuda"), w)
    assert "M=9" in str(e.value)
    # fp32 x is accepted (it is digitised like fp16/bf16 x); an unknown dtype code is not
    y32 = m.gemv_noalloc(x.cuda().float(), w)
    assert torch.equal(y32, m.gemv_noalloc(x.cuda(), w))
    y = torch.empty((1, w.N), device="cuda")
    with pytest.raises(m.BQError) as e:
        m._check(m.lib().bq_gemv_noalloc(x.cuda().data_ptr(), 5, 1, w.c, y.data_ptr(), 2, m._stream()))
    assert e.value.status_name == "BQ_ERR_DTYPE"
