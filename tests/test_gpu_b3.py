"""Ternary weights in base-3 storage (26 bytes per group of 128, 1.75 bits per weight) on the
GPU against the CPU oracle: the device pack is byte-for-byte the oracle's, the unpack reports
the same invalid bytes, the GEMV stays within max|y - y_ref| <= 2e-3 * sum_k |x s| per output on
the integer tensor-core kernel (K a multiple of 1024) and on the SIMT kernel (any K), and the
embedding gather is bit-exact after the same rounding. The full-size matrix (N = 20480,
K = 5120) is checked on sampled rows, launched as the benchmark launches it."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import assert_within_bound, bq, requires_gpu, sample_rows, ternary_q, x_dtype_code

pytestmark = requires_gpu
T3 = oracle.TERNARY_B3


def _pack_both(orc, q, s):
    m = bq()
    w = m.pack_ternary_b3_g128(q.cuda(), s.cuda())
    st, ref, s_ref = orc.pack(T3, q.numpy(), s.numpy())
    assert st == oracle.OK
    return w, ref, s_ref


@pytest.mark.parametrize("N,K", [(1, 128), (3, 1152), (77, 640), (1000, 5120), (33, 2176)])
def test_pack_b3_bit_exact(orc, N, K):
    q = ternary_q(300 + N, N, K)
    s = synth.scales(300 + N, N, K // 128)
    w, ref, s_ref = _pack_both(orc, q, s)
    assert tuple(w.words.shape) == (N, 26 * K // 128) and w.words.dtype == torch.uint8
    assert np.array_equal(w.words.cpu().numpy(), ref)
    assert np.array_equal(w.scales.cpu().view(torch.int16).numpy().view(np.uint16), s_ref)
    m = bq()
    assert m.packed_bytes(m.TERNARY_B3_G128, N, K) == N * 26 * K // 128
    back, s2 = m.unpack_g128(w)
    assert torch.equal(back.cpu(), q) and torch.equal(s2, w.scales)


def test_pack_b3_rejects_values_outside_the_set():
    m = bq()
    q = torch.zeros((4, 256), dtype=torch.int8)
    q[2, 77] = 2
    with pytest.raises(m.BQError) as e:
        m.pack_ternary_b3_g128(q.cuda(), torch.ones((4, 2), dtype=torch.float16, device="cuda"))
    assert e.value.status_name == "BQ_ERR_INVALID_CODE"


def test_unpack_b3_reports_invalid_bytes(orc):
    """Bytes no base-3 value produces (here 1, written over valid ones) are counted and
    their codes unpack as 0, as in the oracle."""
    m = bq()
    N, K = 5, 1152
    q = ternary_q(7, N, K)
    s = synth.scales(7, N, K // 128)
    w, ref, _ = _pack_both(orc, q, s)
    bad = ref.copy()
    bad[0, 3] = 1           # five-code byte: valid values are ceil(256 v / 243), 1 is not one
    bad[4, 233] = 1         # last four-code byte of the tail block
    w.words.copy_(torch.from_numpy(bad))
    qo, nbad = orc.unpack(T3, bad, K)
    assert nbad == 2
    q_dev = torch.empty((N, K), dtype=torch.int8, device="cuda")
    with pytest.raises(m.BQError) as e:
        m._check(m.lib().bq_unpack_g128(w.c, q_dev.data_ptr(), None, m._stream()))
    assert e.value.status_name == "BQ_ERR_INVALID_CODE" and "2 bytes" in str(e.value)
    assert np.array_equal(q_dev.cpu().numpy(), qo)


def run_b3(orc, seed, N, K, M, xdt=torch.bfloat16, ydt=torch.float32, rows=None, x=None, noalloc=False):
    m = bq()
    q = ternary_q(seed, N, K)
    s = synth.scales(seed, N, K // 128)
    if x is None:
        x = synth.activations(seed, M, K, dtype=xdt)
    w, ref, s_ref = _pack_both(orc, q, s)
    y = (m.gemv_noalloc if noalloc else m.gemv)(x.cuda(), w, out_dtype=ydt)
    torch.cuda.synchronize()
    y_ref, bound = orc.gemv(T3, x, x_dtype_code(x.dtype), ref, s_ref, K, rows=rows)
    yg = y if rows is None else y[:, torch.from_numpy(rows).cuda()]
    return assert_within_bound(yg, y_ref, bound, f"base-3 N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("N,K", [(5, 1024), (333, 2048), (2000, 5120)])
def test_b3_tensor_path_all_outputs(orc, M, N, K):
    """Integer tensor-core kernel (K a multiple of 1024), every M (one to four column sets),
    ragged tile counts."""
    run_b3(orc, 600 + M, N, K, M)


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(1, 128), (77, 640), (40, 1152), (9, 2176)])
def test_b3_simt_all_outputs(orc, M, N, K):
    """SIMT kernel: K not a multiple of 1024, including blocks of fewer than 8 groups."""
    run_b3(orc, 700 + M, N, K, M)


@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_b3_dtypes(orc, xdt, ydt):
    run_b3(orc, 8, 513, 1024, 3, xdt=xdt, ydt=ydt)


def test_b3_k5120_n20480_sampled(orc):
    """The benchmark's base-3 matrix: M=1, K=5120, N=20480 (21.3 MB packed)."""
    run_b3(orc, 0, 20480, 5120, 1, rows=sample_rows(20480, 1500))


@pytest.mark.parametrize("M", [1, 8])
def test_b3_noalloc(orc, M):
    run_b3(orc, 9, 700, 5120, M, noalloc=True)


@pytest.mark.parametrize("M", [3, 8])
def test_b3_wide_dynamic_range(orc, M):
    """x spanning 40 binades inside each group: the level combinations x_{i-1} - 3 x_i carried
    as integers 20 bits below the group maximum stay within the bound."""
    K = 2048
    x = synth.activations(7, M, K, dtype=torch.float32)
    mag = torch.tensor([2.0 ** (-30 + (k % 41)) for k in range(K)])
    run_b3(orc, 10, 300, K, M, x=(x * mag).to(torch.bfloat16))


def test_b3_zero_and_tiny_groups(orc):
    K = 1024
    x = synth.activations(8, 4, K).float()
    x[0, :128] = 0.0
    x[1, 128:256] = 1e-30
    x[2, 256:384] = 65504.0
    run_b3(orc, 11, 200, K, 4, x=x.to(torch.float16))


def test_b3_special_codes(orc):
    """All codes -1, all 0, all +1 and alternating rows: the byte extremes (0, 128/127,
    255/253) through the decode."""
    m = bq()
    N, K, M = 64, 2048, 2
    q = torch.empty((N, K), dtype=torch.int8)
    q[0::4] = -1
    q[1::4] = 0
    q[2::4] = 1
    q[3::4] = torch.tensor([(-1, 0, 1)[k % 3] for k in range(K)], dtype=torch.int8)
    s = synth.scales(12, N, K // 128)
    x = synth.activations(12, M, K)
    w, ref, s_ref = _pack_both(orc, q, s)
    y = m.gemv(x.cuda(), w)
    y_ref, bound = orc.gemv(T3, x, oracle.X_BF16, ref, s_ref, K)
    assert_within_bound(y, y_ref, bound, "special codes")
    # all-zero codes: exact integer column sums that cancel only across the digit columns, so
    # the fp32 combination leaves rounding far below the bound (not an exact 0 as with 2 bits)
    z = y[:, 1::4].double().abs().cpu().numpy()
    assert np.all(z <= 1e-3 * bound[:, 1::4])


@pytest.mark.parametrize("M,K,kernel", [(3, 2048, "tensor-core"), (6, 2048, "tensor-core"), (3, 640, "simt")])
def test_b3_nonfinite_x_propagates(orc, M, K, kernel):
    m = bq()
    N = 300
    q = ternary_q(13, N, K)
    s = synth.scales(13, N, K // 128)
    w, ref, s_ref = _pack_both(orc, q, s)
    x = synth.activations(14, M, K)
    x[0, 17] = float("nan")
    x[1, K - 1] = float("inf")
    x[2, 300] = float("-inf")
    y = m.gemv(x.cuda(), w).double().cpu().numpy()
    y_ref, bound = orc.gemv(T3, x, oracle.X_BF16, ref, s_ref, K)
    for t in range(3):
        assert not np.isfinite(y_ref[t]).any() and not np.isfinite(y[t]).any(), f"{kernel}: token {t}"
    assert np.all(np.abs(y[3:] - y_ref[3:]) <= bound[3:])


def test_b3_same_results_as_2bit_within_bound(orc):
    """The same codes in 2-bit and in base-3 storage give outputs within the bound of each
    other's oracle (the oracle gives both the same y, bit for bit)."""
    m = bq()
    N, K, M = 4096, 5120, 4
    q = ternary_q(15, N, K)
    s = synth.scales(15, N, K // 128)
    x = synth.activations(15, M, K).cuda()
    w3 = m.pack_ternary_b3_g128(q.cuda(), s.cuda())
    w2 = m.pack_ternary_g128(q.cuda(), s.cuda())
    y3 = m.gemv(x, w3).double().cpu().numpy()
    y2 = m.gemv(x, w2).double().cpu().numpy()
    rows = sample_rows(N, 300, 15)
    _, ref, s_ref = orc.pack(T3, q.numpy(), s.numpy())
    _, bound = orc.gemv(T3, x.cpu(), oracle.X_BF16, ref, s_ref, K, rows=rows)
    assert np.all(np.abs(y3[:, rows] - y2[:, rows]) <= 2 * bound)


@pytest.mark.parametrize("ot", [torch.bfloat16, torch.float16, torch.float32])
def test_b3_embed(orc, ot):
    m = bq()
    N, K, T = 1000, 1152, 77
    q = ternary_q(16, N, K)
    s = synth.scales(16, N, K // 128)
    w, ref, s_ref = _pack_both(orc, q, s)
    ids = synth.random_ids(16, synth.TID_IDS, T, N)
    out = m.embed_gather(ids.cuda(), w, out_dtype=ot).cpu()
    exp, bad = orc.embed(T3, ids.numpy(), ref, s_ref, K)
    assert bad == 0
    if ot == torch.float32:
        assert np.array_equal(out.numpy().astype(np.float64), exp)
    else:
        e = orc.to_bf16_bits(exp) if ot == torch.bfloat16 else exp.astype(np.float16).view(np.uint16)
        ev = torch.from_numpy(e.view(np.int16)).view(ot).float()
        assert torch.equal(out.float(), ev)


def run_b3_prefill(orc, seed, M, N, K, xdt=torch.bfloat16, ydt=torch.float32, rows=None, x=None):
    m = bq()
    q = ternary_q(seed, N, K)
    s = synth.scales(seed, N, K // 128)
    w, ref, s_ref = _pack_both(orc, q, s)
    if x is None:
        x = synth.activations(seed + 1, M, K, dtype=xdt)
    y = m.gemm_prefill(x.cuda(), w, out_dtype=ydt)
    torch.cuda.synchronize()
    m.get_device_error()
    y_ref, bound = orc.gemv(T3, x, x_dtype_code(x.dtype), ref, s_ref, K, rows=rows)
    yg = y if rows is None else y[:, torch.from_numpy(rows).cuda()]
    return assert_within_bound(yg, y_ref, bound, f"base-3 prefill M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (17, 300, 640), (77, 1000, 256), (130, 256, 1152),
                                   (300, 200, 2176), (512, 384, 5120)])
def test_b3_prefill_all_outputs(orc, M, N, K):
    """tcgen05 prefill with the base-3 operand expansion: all four 32-weight parts of a group,
    blocks of fewer than 8 groups, split tails."""
    run_b3_prefill(orc, 800 + M, M, N, K)


@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("xdt", [torch.float16, torch.bfloat16])
def test_b3_prefill_dtypes(orc, xdt, ydt):
    run_b3_prefill(orc, 18, 200, 256, 1024, xdt=xdt, ydt=ydt)


def test_b3_prefill_m512_k5120_n20480_sampled(orc):
    """The ternary prefill workload (M=512, K=5120, N=20480) in base-3 storage, all tokens of
    sampled weight rows, launched as the benchmark launches it."""
    run_b3_prefill(orc, 0, 512, 20480, 5120, rows=sample_rows(20480, 400))


def test_b3_prefill_special_codes(orc):
    """Rows of all -1, all 0, all +1 codes and a repeating pattern through the prefill decode."""
    m = bq()
    N, K, M = 128, 1024, 64
    q = torch.empty((N, K), dtype=torch.int8)
    q[0::4] = -1
    q[1::4] = 0
    q[2::4] = 1
    q[3::4] = torch.tensor([(-1, 0, 1)[k % 3] for k in range(K)], dtype=torch.int8)
    s = synth.scales(19, N, K // 128)
    x = synth.activations(19, M, K)
    w, ref, s_ref = _pack_both(orc, q, s)
    y = m.gemm_prefill(x.cuda(), w)
    y_ref, bound = orc.gemv(T3, x, oracle.X_BF16, ref, s_ref, K)
    assert_within_bound(y, y_ref, bound, "prefill special codes")
    assert torch.all(y[:, 1::4] == 0)
