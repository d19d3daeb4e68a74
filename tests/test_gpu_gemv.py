"""GPU decode GEMV against the CPU oracle, within max|y - y_ref| <= 2e-3 * sum_k |x s| per
output. Small shapes are checked on every output; the full-size workloads (K = 5120 with
N = 5120 / 20480, the 248 320-row LM head, the ternary N = 20480 matrix) on the first and
last rows plus a seeded sample, launched exactly as the benchmark launches them."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import (assert_within_bound, binary_inputs, bq, requires_gpu, sample_rows,
                              ternary_q, x_dtype_code)

pytestmark = requires_gpu


def run_binary(orc, seed, N, K, M, xdt=torch.bfloat16, ydt=torch.float32, rows=None):
    m = bq()
    x, words, s = binary_inputs(seed, N, K, M, xdt)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    y = m.gemv(x.cuda(), w, out_dtype=ydt)
    torch.cuda.synchronize()
    r = None if rows is None else rows
    y_ref, bound = orc.gemv(oracle.BINARY, x, x_dtype_code(xdt), words, s, K, rows=r)
    yg = y if r is None else y[:, torch.from_numpy(r).cuda()]
    return assert_within_bound(yg, y_ref, bound, f"binary N={N} K={K} M={M}")


def test_config_1024_fp16_seed0(orc):
    """Binary GEMV, M=1, K=N=1024, x fp16, seed 0 -- every output."""
    run_binary(orc, 0, 1024, 1024, 1, xdt=torch.float16)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("N,K", [(1, 128), (7, 256), (33, 1152), (1000, 640), (9120, 384)])
def test_binary_ragged_all_outputs(orc, M, N, K):
    run_binary(orc, 100 + M, N, K, M)


@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_binary_dtypes(orc, xdt, ydt):
    run_binary(orc, 7, 513, 1024, 3, xdt=xdt, ydt=ydt)


@pytest.mark.parametrize("M", [1, 4, 8])
def test_binary_k5120_n5120_all_outputs(orc, M):
    run_binary(orc, 0, 5120, 5120, M)


@pytest.mark.parametrize("M", [1, 4, 8])
def test_binary_k5120_n20480_sampled(orc, M):
    run_binary(orc, 0, 20480, 5120, M, rows=sample_rows(20480, 1500, M))


@pytest.mark.parametrize("N,K", [(9120, 5120), (40960, 5120), (5120, 20480)])
def test_full_depth_block_shapes_sampled(orc, N, K):
    """The shapes of one block of the full-depth decode step (attention in, MLP gate/up,
    MLP down; attention out is the 5120 x 5120 case above), M=1, as the step launches them."""
    run_binary(orc, 64, N, K, 1, rows=sample_rows(N, 800, 1))


def test_binary_lm_head_sampled(orc):
    """LM head: M=1, K=5120, N=248320 (~159 MB packed + ~20 MB scales)."""
    run_binary(orc, 0, 248320, 5120, 1, rows=sample_rows(248320, 1500))


def run_ternary(orc, seed, N, K, M, xdt=torch.bfloat16, ydt=torch.float32, rows=None):
    m = bq()
    q = ternary_q(seed, N, K)
    s = synth.scales(seed, N, K // 128)
    x = synth.activations(seed, M, K, dtype=xdt)
    w = m.pack_ternary_g128(q.cuda(), s.cuda())
    y = m.gemv(x.cuda(), w, out_dtype=ydt)
    torch.cuda.synchronize()
    st, words_ref, s_ref = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
    assert st == oracle.OK
    y_ref, bound = orc.gemv(oracle.TERNARY, x, x_dtype_code(xdt), words_ref, s_ref, K, rows=rows)
    yg = y if rows is None else y[:, torch.from_numpy(rows).cuda()]
    return assert_within_bound(yg, y_ref, bound, f"ternary N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(1, 128), (45, 640), (1000, 1152)])
def test_ternary_ragged_all_outputs(orc, M, N, K):
    run_ternary(orc, 200 + M, N, K, M)


def test_ternary_k5120_n20480_sampled(orc):
    run_ternary(orc, 0, 20480, 5120, 1, rows=sample_rows(20480, 1500))


def test_ternary_fp16_x(orc):
    run_ternary(orc, 3, 300, 1024, 2, xdt=torch.float16, ydt=torch.bfloat16)


def test_special_weights(orc):
    """All-ones and all-zero rows, and a ternary all-zero-code row, on the GPU."""
    m = bq()
    N, K, M = 3, 512, 2
    x = synth.activations(5, M, K)
    s = synth.scales(5, N, K // 128)
    s[1] = s[0]                                    # rows 0 and 1 share their scales
    words = torch.zeros((N, K // 32), dtype=torch.int32)
    words[0] = -1                                  # every bit 1 -> +s; rows 1, 2: every bit 0
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    y = m.gemv(x.cuda(), w).cpu()
    y_ref, bound = orc.gemv(oracle.BINARY, x, oracle.X_BF16, words, s, K)
    assert_within_bound(y, y_ref, bound)
    assert torch.allclose(y[:, 0], -y[:, 1], rtol=0, atol=1e-6)
    tw = torch.full((N, K // 16), 0x55555555, dtype=torch.int32)
    wt = m.BQWeight(m.TERNARY_G128, N, K, tw.cuda(), s.cuda())
    yt = m.gemv(x.cuda(), wt).cpu()
    assert torch.all(yt == 0)


def test_api_errors_on_device():
    m = bq()
    N, K = 16, 256
    x, words, s = binary_inputs(1, N, K, 2)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    xd = x.cuda()
    with pytest.raises(m.BQError) as e:
        m.gemv(torch.empty((9, K), dtype=torch.bfloat16, device="cuda"), w)
    assert e.value.status_name == "BQ_ERR_SHAPE"
    buf = torch.empty(2 * K + 1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BQError) as e:
        m.gemv(buf[1:].view(2, K), w)                         # 2-byte offset: misaligned
    assert e.value.status_name == "BQ_ERR_ALIGNMENT"
    m.gemv(xd, w)                                              # still works afterwards
    torch.cuda.synchronize()


# ---- tensor-core path (K a multiple of 1024): fp8 pieces of x, stream-K split ----------

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,K", [(1, 1024), (127, 2048), (129, 1024), (1000, 3072)])
def test_tensor_path_ragged_all_outputs(orc, M, xdt, N, K):
    """All outputs of ragged shapes on the tensor-core kernels: mma.sync for M <= 4, tcgen05
    (sign operand in tensor memory) for binary M >= 5."""
    run_binary(orc, 400 + M, N, K, M, xdt=xdt)


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("N,K", [(5, 1024), (333, 2048), (2000, 5120)])
def test_tensor_path_ternary(orc, M, N, K):
    run_ternary(orc, 500 + M, N, K, M)


@pytest.mark.parametrize("M", [3, 8])
def test_tensor_path_wide_dynamic_range(orc, M):
    """x spanning 40 binades inside each group: the integer digits of x (22 bits below the
    group maximum) stay within the bound. M = 3 runs the mma.sync kernel, M = 8 the tcgen05 one."""
    m = bq()
    N, K = 300, 2048
    x = synth.activations(7, M, K, dtype=torch.float32)
    mag = torch.tensor([2.0 ** (-30 + (k % 41)) for k in range(K)])
    x = (x * mag).to(torch.bfloat16)
    words = synth.binary_words(7, N, K)
    s = synth.scales(7, N, K // 128)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    y = m.gemv(x.cuda(), w)
    y_ref, bound = orc.gemv(oracle.BINARY, x, oracle.X_BF16, words, s, K)
    assert_within_bound(y, y_ref, bound, "wide range")


@pytest.mark.parametrize("M", [2, 6])
def test_tensor_path_zero_and_tiny_groups(orc, M):
    m = bq()
    N, K = 200, 1024
    x = synth.activations(8, M, K).float()
    x[0, :128] = 0.0                                   # an all-zero group
    x[1, 128:256] = 1e-30                              # a group of tiny values
    x = x.to(torch.bfloat16)
    words = synth.binary_words(8, N, K)
    s = synth.scales(8, N, K // 128)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    y = m.gemv(x.cuda(), w)
    y_ref, bound = orc.gemv(oracle.BINARY, x, oracle.X_BF16, words, s, K)
    assert_within_bound(y, y_ref, bound, "zero/tiny groups")


def test_tensor_path_deterministic():
    """Split blocks are summed in a fixed order: repeated calls give identical bits."""
    m = bq()
    x, words, s = binary_inputs(9, 5120, 5120, 8)
    w = m.BQWeight(m.BINARY_G128, 5120, 5120, words.cuda(), s.cuda())
    xd = x.cuda()
    y1 = m.gemv(xd, w).clone()
    for _ in range(5):
        assert torch.equal(m.gemv(xd, w), y1)


def test_workspace_too_small_is_rejected():
    m = bq()
    x, words, s = binary_inputs(10, 256, 1024, 2)
    w = m.BQWeight(m.BINARY_G128, 256, 1024, words.cuda(), s.cuda())
    need = m.gemv_workspace_bytes(2, w)
    assert need > 0
    y = torch.empty((2, 256), dtype=torch.float32, device="cuda")
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.BQError) as e:
        m._check(m.lib().bq_gemv(x.cuda().data_ptr(), 1, 2, w.c, y.data_ptr(), 2, ws.data_ptr(),
                                 need - 256, m._stream()))
    assert e.value.status_name == "BQ_ERR_WORKSPACE"
