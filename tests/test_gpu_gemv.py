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


# ---- tensor-core path (K a multiple of 1024): x as integer digits, whole rows per CTA ------

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,K", [(1, 1024), (127, 2048), (129, 1024), (1000, 3072)])
def test_tensor_path_ragged_all_outputs(orc, M, xdt, N, K):
    """All outputs of ragged shapes on the integer tensor-core kernel, every M (one to four
    column sets), tile counts that leave partial tile-groups, both x types."""
    run_binary(orc, 400 + M, N, K, M, xdt=xdt)


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("N,K", [(5, 1024), (333, 2048), (2000, 5120)])
def test_tensor_path_ternary(orc, M, N, K):
    run_ternary(orc, 500 + M, N, K, M)


@pytest.mark.parametrize("M", [3, 8])
def test_tensor_path_wide_dynamic_range(orc, M):
    """x spanning 40 binades inside each group: the integer digits of x (22 bits below the
    group maximum) stay within the bound, at two and at four column sets."""
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
    """The eight per-group sums of every output are added in a fixed order: repeated calls
    give identical bits."""
    m = bq()
    x, words, s = binary_inputs(9, 5120, 5120, 8)
    w = m.BQWeight(m.BINARY_G128, 5120, 5120, words.cuda(), s.cuda())
    xd = x.cuda()
    y1 = m.gemv(xd, w).clone()
    for _ in range(5):
        assert torch.equal(m.gemv(xd, w), y1)


def test_workspace_sizes():
    """The tensor-core path keeps the digit fragments of x in the workspace (written once per
    call by the prep kernel; 1 KB per group and column set, plus factors and accumulator
    inputs), the SIMT path needs none, and a workspace that is too small is rejected before
    anything is launched."""
    m = bq()
    x, words, s = binary_inputs(10, 256, 1024, 4)
    w = m.BQWeight(m.BINARY_G128, 256, 1024, words.cuda(), s.cuda())
    assert m.gemv_workspace_bytes(1, w) >= 8 * 1024
    w640 = m.BQWeight(m.BINARY_G128, 256, 640, synth.binary_words(10, 256, 640).cuda(),
                      synth.scales(10, 256, 5).cuda())
    assert m.gemv_workspace_bytes(4, w640) == 0
    need = m.gemv_workspace_bytes(4, w)
    assert need > 0
    y = torch.empty((4, 256), dtype=torch.float32, device="cuda")
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.BQError) as e:
        m._check(m.lib().bq_gemv(x.cuda().data_ptr(), 1, 4, w.c, y.data_ptr(), 2, ws.data_ptr(),
                                 need - 256, m._stream()))
    assert e.value.status_name == "BQ_ERR_WORKSPACE"


@pytest.mark.parametrize("M,K,kernel", [(3, 2048, "tensor-core"), (6, 2048, "tensor-core"), (3, 640, "simt")])
@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY])
def test_nonfinite_x_propagates(orc, M, K, kernel, fmt):
    """An infinity or NaN in x makes every output of that token non-finite, as in the oracle
    (the tensor-core kernel gives NaN: the digit prep marks the group's factor NaN); tokens
    with finite x are unaffected. K = 2048 runs the integer tensor-core kernel (two and four
    column sets), K = 640 the SIMT kernel."""
    m = bq()
    N = 700
    s = synth.scales(5, N, K // 128)
    if fmt == oracle.BINARY:
        words = synth.binary_words(5, N, K)
        w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
        words_np = words.numpy()
    else:
        q = ternary_q(5, N, K)
        w = m.pack_ternary_g128(q.cuda(), s.cuda())
        st, words_np, _ = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
        assert st == oracle.OK
    x = synth.activations(6, M, K)
    x[0, 17] = float("nan")
    x[1, K - 1] = float("inf")
    x[2, 300] = float("-inf")
    y = m.gemv(x.cuda(), w).double().cpu().numpy()
    torch.cuda.synchronize()
    y_ref, bound = orc.gemv(fmt, x, oracle.X_BF16, words_np, s, K)
    for t in range(3):
        assert not np.isfinite(y_ref[t]).any(), "the oracle's outputs of that token are non-finite"
        assert not np.isfinite(y[t]).any(), f"{kernel}: token {t} has finite outputs"
    err = np.abs(y[3:] - y_ref[3:])
    assert np.all(err <= bound[3:]), f"{kernel}: finite tokens, max err/bound {np.max(err / bound[3:]):.3g}"


def test_binding_rejects_wrong_out_shape():
    """The binding checks a caller's out tensor (shape, dtype, device) before anything is
    launched: a smaller out would otherwise receive out-of-bounds writes."""
    m = bq()
    N, K = 64, 1024
    x, words, s = binary_inputs(2, N, K, 3)
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    xd = x.cuda()
    for bad in (torch.empty((3, N - 1), device="cuda"), torch.empty((2, N), device="cuda"),
                torch.empty((3, N), dtype=torch.int32, device="cuda"), torch.empty((3, N))):
        with pytest.raises(ValueError):
            m.gemv(xd, w, out=bad)
        with pytest.raises(ValueError):
            m.gemv_noalloc(xd, w, out=bad)
        with pytest.raises(ValueError):
            m.gemm_prefill(xd, w, out=bad)
    with pytest.raises(ValueError):
        m.gemv(x, w)                                            # x on the host
