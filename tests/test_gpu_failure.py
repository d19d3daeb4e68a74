"""Failure paths on the GPU, in forms that fault, trap or hang nothing:

* a bounded pipeline wait that runs out: the test hook bq_debug_set_wait_limit_ns makes the
  GEMV's and the prefill's pipeline waits give up after 1 ns, so that waits for stages that
  are still in flight time out. The kernels then record BQ_ERR_TIMEOUT, drain their copies and
  MMAs (those waits keep the 2 s limit), free tensor memory and return; bq_get_device_error
  reports the timeout once, and the next normal calls are correct (checked against the oracle).
* an injected launch failure (host side): BQ_ERR_CUDA with nothing launched, after which calls
  work again."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import assert_within_bound, bq, requires_gpu, sample_rows

pytestmark = requires_gpu


def _binary(m, seed, N, K):
    words = synth.binary_words(seed, N, K)
    s = synth.scales(seed, N, K // 128)
    return m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda()), words, s


def test_wait_timeout_reported_then_recovers(orc):
    m = bq()
    N, K = 20480, 5120
    w, words, s = _binary(m, 41, N, K)
    x = synth.activations(42, 4, K)
    xp = synth.activations(43, 512, K)
    xd, xpd = x.cuda(), xp.cuda()
    m.get_device_error()                                    # nothing pending
    m.debug_set_wait_limit_ns(1)
    try:
        for call in (lambda: m.gemv(xd, w), lambda: m.gemm_prefill(xpd, w)):
            call()
            torch.cuda.synchronize()
            with pytest.raises(m.BQError) as e:
                m.get_device_error()
            assert e.value.status_name == "BQ_ERR_TIMEOUT"
            m.get_device_error()                            # read once, then cleared
    finally:
        m.debug_set_wait_limit_ns(0)
    # the context is usable and the kernels are correct again
    rows = sample_rows(N, 300, 3)
    y = m.gemv(xd, w)
    yp = m.gemm_prefill(xpd, w)
    torch.cuda.synchronize()
    m.get_device_error()
    ref, bound = orc.gemv(oracle.BINARY, x, oracle.X_BF16, words, s, K, rows=rows)
    assert_within_bound(y[:, torch.from_numpy(rows).cuda()], ref, bound, "gemv after a timeout")
    ref, bound = orc.gemv(oracle.BINARY, xp, oracle.X_BF16, words, s, K, rows=rows[:40])
    assert_within_bound(yp[:, torch.from_numpy(rows[:40]).cuda()], ref, bound, "prefill after a timeout")


def test_injected_launch_failure_then_recovers(orc):
    m = bq()
    N, K = 1000, 2048
    w, words, s = _binary(m, 44, N, K)
    x = synth.activations(45, 2, K)
    xd = x.cuda()
    y = torch.full((2, N), 7.0, device="cuda")
    m.debug_fail_next_launches(1)
    try:
        with pytest.raises(m.BQError) as e:
            m.gemv(xd, w, out=y)
        assert e.value.status_name == "BQ_ERR_CUDA" and "injected" in str(e.value)
        torch.cuda.synchronize()
        assert torch.all(y == 7.0)                          # nothing ran
    finally:
        m.debug_fail_next_launches(0)
    m.gemv(xd, w, out=y)
    torch.cuda.synchronize()
    ref, bound = orc.gemv(oracle.BINARY, x, oracle.X_BF16, words, s, K)
    assert_within_bound(y, ref, bound, "gemv after an injected failure")


def test_wait_timeout_in_topk_and_mlp_then_recovers(orc):
    """The same bounded-wait timeout in the top-k GEMV (its CTAs still take their tickets and the
    last one still merges, so nothing waits forever) and in the SwiGLU MLP's two GEMVs; then
    normal calls are correct."""
    m = bq()
    N, K, F = 20480, 5120, 2048
    w, words, s = _binary(m, 51, N, K)
    g, gw, gs = _binary(m, 52, F, K)
    u, uw, us = _binary(m, 53, F, K)
    d, dw, ds = _binary(m, 54, 1024, F)
    x = synth.activations(55, 2, K)
    xd = x.cuda()
    m.get_device_error()
    m.debug_set_wait_limit_ns(1)
    try:
        for call in (lambda: m.gemv_topk(xd, w, k=20), lambda: m.mlp_swiglu(xd, g, u, d)):
            call()
            torch.cuda.synchronize()
            with pytest.raises(m.BQError) as e:
                m.get_device_error()
            assert e.value.status_name == "BQ_ERR_TIMEOUT"
            m.get_device_error()
    finally:
        m.debug_set_wait_limit_ns(0)
    vals, idx = m.gemv_topk(xd, w, k=20)
    y = m.mlp_swiglu(xd, g, u, d)
    torch.cuda.synchronize()
    m.get_device_error()
    yl = m.gemv(xd, w).cpu().numpy()
    order = np.array([np.lexsort((np.arange(N), -r.astype(np.float64)))[:20] for r in yl])
    assert np.array_equal(idx.cpu().numpy(), order)
    _, y_ref, bound = orc.mlp_swiglu(x, oracle.X_BF16, oracle.BINARY, (gw.numpy(), gs), (uw.numpy(), us),
                                     oracle.BINARY, (dw.numpy(), ds))
    assert_within_bound(y, y_ref, bound, "mlp after a timeout")
