"""GPU prefill GEMM (tcgen05) against the CPU oracle, within 2e-3 * sum_k |x s| per output.
Small ragged shapes are checked on every output; the M=512, K=5120, N=20480 binary and
ternary workloads on sampled weight rows (all 512 tokens), launched as the benchmark
launches them."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import (assert_within_bound, bq, requires_gpu, sample_rows, ternary_q,
                              x_dtype_code)

pytestmark = requires_gpu


def weight(m, fmt, seed, N, K):
    s = synth.scales(seed, N, K // 128)
    if fmt == oracle.BINARY:
        words = synth.binary_words(seed, N, K)
        return m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda()), words.numpy(), s
    q = ternary_q(seed, N, K)
    w = m.pack_ternary_g128(q.cuda(), s.cuda())
    return w, w.words.cpu().numpy(), s


def check(orc, fmt, seed, M, N, K, xdt=torch.bfloat16, ydt=torch.float32, rows=None):
    m = bq()
    w, words_np, s = weight(m, fmt, seed, N, K)
    if fmt == oracle.TERNARY:
        # the oracle packs the same q itself; the device words must agree bit for bit
        q = ternary_q(seed, N, K)
        st, words_ref, _ = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
        assert np.array_equal(words_np.view(np.uint32), words_ref)
        words_np = words_ref
    x = synth.activations(seed + 1, M, K, dtype=xdt)
    y = m.gemm_prefill(x.cuda(), w, out_dtype=ydt)
    torch.cuda.synchronize()
    m.get_device_error()
    y_ref, bound = orc.gemv(fmt, x, x_dtype_code(xdt), words_np, s, K, rows=rows)
    yg = y if rows is None else y[:, torch.from_numpy(rows).cuda()]
    return assert_within_bound(yg, y_ref, bound, f"prefill fmt={fmt} M={M} N={N} K={K}")


@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY])
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (17, 300, 640), (77, 1000, 256), (64, 129, 384),
                                   (130, 256, 1152), (300, 200, 512), (512, 384, 640)])
def test_prefill_ragged_all_outputs(orc, fmt, M, N, K):
    check(orc, fmt, 300 + M, M, N, K)


@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_prefill_dtypes(orc, xdt, ydt):
    check(orc, oracle.BINARY, 9, 200, 256, 1024, xdt=xdt, ydt=ydt)


@pytest.mark.parametrize("N,ydt", [(1000, torch.bfloat16), (1000, torch.float16), (300, torch.bfloat16),
                                   (129, torch.float32), (392, torch.float32)])
def test_prefill_output_store_paths(orc, N, ydt):
    """Rows of Y that are a whole number of 16-byte units leave each tile as one tensor-map
    store clipped at M and N (N = 1000, 392); other widths take per-row stores (N = 300 in a
    16-bit type, N = 129 in fp32). Ragged M = 77 clips the token side of the box."""
    check(orc, oracle.BINARY, 31, 77, N, 512, ydt=ydt)


@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY])
def test_prefill_m512_k5120_n20480_sampled(orc, fmt):
    check(orc, fmt, 0, 512, 20480, 5120, rows=sample_rows(20480, 96, 5))


@pytest.mark.parametrize("fmt,M", [(oracle.BINARY, 128), (oracle.TERNARY, 77)])
def test_prefill_split_tail_rows(orc, fmt, M):
    """160 tiles of 128 rows on 148 SMs: the 12 tiles past the full wave are split along K
    (8 splits) and their fp32 partials added in order by a reduce pass. Every row of those
    tiles is checked, plus a sample of the whole-K tiles."""
    N, K = 20480, 2048
    tail_rows = np.arange(148 * 128, N)
    rows = np.unique(np.concatenate([tail_rows, sample_rows(148 * 128, 64, 7)]))
    check(orc, fmt, 21, M, N, K, rows=rows)


@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY])
def test_prefill_m512_split_tail_rows(orc, fmt):
    """M = 512 at BN = 256: 320 tiles of 128 rows on 148 SMs, the 24 past the second full
    wave (rows 18944 .. 20479, both token tiles) split along K and reduced. Every one of
    those rows is checked, plus a sample of the whole-K rows."""
    N, K = 20480, 2048
    tail_rows = np.arange(148 * 128, N)
    rows = np.unique(np.concatenate([tail_rows, sample_rows(N - 16 * 256, 64, 8)]))
    check(orc, fmt, 23, 512, N, K, rows=rows)


def test_prefill_fp16_is_exact_scale(orc):
    """With fp16 x the +-s operand is exact: the error is fp32 accumulation only."""
    r = check(orc, oracle.BINARY, 11, 256, 512, 2048, xdt=torch.float16)
    assert r < 0.05


def test_prefill_matches_gemv(orc):
    """For M <= 8 the prefill kernel and the decode GEMV compute the same product."""
    m = bq()
    w, _, _ = weight(m, oracle.BINARY, 12, 1000, 1024)
    x = synth.activations(13, 8, 1024, dtype=torch.float16).cuda()
    a = m.gemm_prefill(x, w)
    b = m.gemv(x, w)
    assert torch.allclose(a, b, rtol=1e-4, atol=1e-4)


# ---------------------------------------------------------------------------------------
# bf16 x with scales that bf16 cannot hold: the +-s operand must stay exact
# ---------------------------------------------------------------------------------------

from tests.adversarial import (adversarial_binary, adversarial_ternary_q, positive_bf16_x,  # noqa: E402
                               wide_range_bf16_x)


def check_adversarial(orc, fmt, M, N, K, x, rows=None):
    m = bq()
    if fmt == oracle.BINARY:
        words, s = adversarial_binary(N, K)
        w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
        words_np = words.numpy()
    else:
        q, s = adversarial_ternary_q(N, K)
        w = m.pack_ternary_g128(q.cuda(), s.cuda())
        st, words_np, _ = orc.pack(oracle.TERNARY, q.numpy(), s.numpy())
        assert st == oracle.OK
        assert np.array_equal(w.words.cpu().numpy().view(np.uint32), words_np)
    y = m.gemm_prefill(x.cuda(), w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    m.get_device_error()
    y_ref, bound = orc.gemv(fmt, x, oracle.X_BF16, words_np, s, K, rows=rows)
    yg = y if rows is None else y[:, torch.from_numpy(rows).cuda()]
    return assert_within_bound(yg, y_ref, bound, f"adversarial prefill fmt={fmt} M={M} N={N} K={K}")


@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY])
@pytest.mark.parametrize("M", [77, 512])
def test_prefill_bf16_tie_scales_all_outputs(orc, fmt, M):
    """Scales on bf16 rounding ties in many binades (0x3C04 = 1.00390625 rounds to 1.0 in
    bf16, a 2^-8 relative error), groups of all-ones / all-zeros bits (or all +1 / all -1
    ternary codes) and strictly positive bf16 x, so that every term of a group would err the
    same way if the scale were rounded to bf16: about 1.95x the bound. With the exact fp16
    operand only fp32 accumulation error is left. Every output is checked."""
    K, N = 1024, 256
    r = check_adversarial(orc, fmt, M, N, K, positive_bf16_x(40 + M, M, K))
    print(f"max err/bound = {r:.4g}")
    assert r < 0.1


@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY])
def test_prefill_bf16_tie_scales_split_tail(orc, fmt):
    """The same adversarial inputs through the split tail: M = 512, N = 10240, K = 1024 is 160
    tiles on 148 SMs; the 12 tiles past the full wave (rows 9472 .. 10239, both token tiles)
    are split along K and reduced, where the per-token factor is applied by the reduce pass.
    Every row of those tiles and a sample of the others are checked."""
    M, N, K = 512, 10240, 1024
    rows = np.unique(np.concatenate([np.arange(74 * 128, N), sample_rows(74 * 128, 64, 9)]))
    r = check_adversarial(orc, fmt, M, N, K, positive_bf16_x(51, M, K), rows=rows)
    assert r < 0.1


@pytest.mark.parametrize("M,N", [(130, 384), (512, 10240)])
def test_prefill_bf16_wide_range_tokens(orc, M, N):
    """Token rows whose magnitudes span 2^-100 .. 2^100 (two binades per token): each row
    gets its own power-of-two factor, so a factor applied to the wrong token, or one lost in
    the split-tail reduce (M = 512, N = 10240: rows 9472 .. 10239 are split along K), shows
    up at once. Rows of all zeros give zeros."""
    K = 1024
    rows = None if N < 1000 else np.unique(np.concatenate([np.arange(74 * 128, N),
                                                           sample_rows(74 * 128, 32, 10)]))
    r = check_adversarial(orc, oracle.BINARY, M, N, K, wide_range_bf16_x(60, M, K), rows=rows)
    assert r < 0.1
