"""SwiGLU MLP of a decode step on the GPU (gate/up GEMV with the SwiGLU epilogue, then the down
GEMV on its fp32 activations) against the CPU oracle: max|y - y_ref| <= 2e-3 * sum_j |a_j s_down|
per output, a being the oracle's activations. Small shapes are checked on every output; the
block of the full-depth step (gate and up 20480 x 5120, down 5120 x 20480) on sampled rows."""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import assert_within_bound, bq, requires_gpu, sample_rows, ternary_q

pytestmark = requires_gpu


def make(orc, fmt, seed, N, K, tid):
    """(device weight, oracle packed, oracle scales) of a random matrix in format fmt."""
    m = bq()
    s = synth.scales(seed + tid, N, K // 128)
    if fmt == oracle.BINARY:
        words = synth.binary_words(seed + tid, N, K)
        return m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda()), words.numpy(), s
    q = synth.random_ternary(seed + tid, synth.TID_TERNARY, (N, K))
    w = (m.pack_ternary_g128 if fmt == oracle.TERNARY else m.pack_ternary_b3_g128)(q.cuda(), s.cuda())
    st, ref, s_ref = orc.pack(fmt, q.numpy(), s.numpy())
    assert st == oracle.OK
    return w, ref, s_ref


def run(orc, fmt_gu, fmt_d, seed, M, K, F, N, xdt=torch.bfloat16, ydt=torch.float32, rows=None):
    m = bq()
    wg, pg, sg = make(orc, fmt_gu, seed, F, K, 1)
    wu, pu, su = make(orc, fmt_gu, seed, F, K, 2)
    wd, pd, sd = make(orc, fmt_d, seed, N, F, 3)
    x = synth.activations(seed, M, K, dtype=xdt)
    y = m.mlp_swiglu(x.cuda(), wg, wu, wd, out_dtype=ydt)
    torch.cuda.synchronize()
    a, y_ref, bound = orc.mlp_swiglu(x, oracle.X_F16 if xdt == torch.float16 else oracle.X_BF16, fmt_gu,
                                     (pg, sg), (pu, su), fmt_d, (pd, sd))
    if rows is not None:
        y_ref, bound, y = y_ref[:, rows], bound[:, rows], y[:, torch.from_numpy(rows).cuda()]
    return assert_within_bound(y, y_ref, bound, f"mlp gu={fmt_gu} d={fmt_d} M={M} K={K} F={F} N={N}")


@pytest.mark.parametrize("M", [1, 2, 5, 8])
@pytest.mark.parametrize("fmt_gu,fmt_d", [(oracle.BINARY, oracle.BINARY), (oracle.TERNARY, oracle.BINARY),
                                          (oracle.TERNARY_B3, oracle.TERNARY)])
def test_mlp_small_all_outputs(orc, fmt_gu, fmt_d, M):
    run(orc, fmt_gu, fmt_d, 100 + M, M, 1024, 1024, 512)


@pytest.mark.parametrize("F", [128, 1152, 4224])
def test_mlp_down_any_k(orc, F):
    """Gate/up row counts (= the down K) that are not a multiple of 1024: the down GEMV takes the
    SIMT kernel on the fp32 activations; a single gate/up pair (F = 128)."""
    run(orc, oracle.BINARY, oracle.BINARY, 200, 3, 2048, F, 300)


@pytest.mark.parametrize("xdt,ydt", [(torch.float16, torch.bfloat16), (torch.float32, torch.float16)])
def test_mlp_dtypes(orc, xdt, ydt):
    m = bq()
    if xdt == torch.float32:
        # fp32 x: compare with the oracle on the same values rounded to bf16 (exactly representable)
        x16 = synth.activations(3, 2, 1024, dtype=torch.bfloat16)
        wg, pg, sg = make(orc, oracle.BINARY, 3, 512, 1024, 1)
        wu, pu, su = make(orc, oracle.BINARY, 3, 512, 1024, 2)
        wd, pd, sd = make(orc, oracle.BINARY, 3, 256, 512, 3)
        y = m.mlp_swiglu(x16.float().cuda(), wg, wu, wd, out_dtype=ydt)
        a, y_ref, bound = orc.mlp_swiglu(x16, oracle.X_BF16, oracle.BINARY, (pg, sg), (pu, su), oracle.BINARY,
                                         (pd, sd))
        assert_within_bound(y, y_ref, bound, "fp32 x")
    else:
        run(orc, oracle.BINARY, oracle.TERNARY, 4, 3, 1024, 512, 256, xdt=xdt, ydt=ydt)


def test_mlp_full_block_sampled(orc):
    """The MLP of one block of the full-depth step at M = 1: gate and up 20480 x 5120, down
    5120 x 20480, binary."""
    run(orc, oracle.BINARY, oracle.BINARY, 0, 1, 5120, 20480, 5120, rows=sample_rows(5120, 600))


def test_mlp_matches_separate_calls(orc):
    """The fused call equals, within the bound, three separate GEMVs with SwiGLU applied in
    between by torch on the fp32 gate and up outputs."""
    m = bq()
    M, K, F, N = 4, 2048, 2048, 1024
    wg, pg, sg = make(orc, oracle.TERNARY, 7, F, K, 1)
    wu, pu, su = make(orc, oracle.TERNARY, 7, F, K, 2)
    wd, pd, sd = make(orc, oracle.BINARY, 7, N, F, 3)
    x = synth.activations(7, M, K).cuda()
    y = m.mlp_swiglu(x, wg, wu, wd)
    g = m.gemv(x, wg)
    u = m.gemv(x, wu)
    a = (g * torch.sigmoid(g) * u).contiguous()
    y2 = m.gemv(a, wd)
    _, y_ref, bound = orc.mlp_swiglu(x.cpu(), oracle.X_BF16, oracle.TERNARY, (pg, sg), (pu, su), oracle.BINARY,
                                     (pd, sd))
    diff = (y - y2).abs().double().cpu().numpy()
    assert np.all(diff <= bound)


def test_mlp_errors():
    m = bq()
    K, F = 1024, 512
    w = lambda N, K_: m.BQWeight(m.BINARY_G128, N, K_, synth.binary_words(1, N, K_).cuda(),
                                 synth.scales(1, N, K_ // 128).cuda())
    x = synth.activations(1, 1, K).cuda()
    with pytest.raises(m.BQError) as e:
        m.mlp_swiglu(x, w(F, K), w(F + 16, K), w(256, F))            # gate and up differ
    assert e.value.status_name == "BQ_ERR_SHAPE"
    with pytest.raises(m.BQError) as e:
        m.mlp_swiglu(x, w(F, K), w(F, K), w(256, F + 128))           # down K != F
    assert e.value.status_name == "BQ_ERR_SHAPE"
    x640 = synth.activations(1, 1, 640).cuda()
    with pytest.raises(m.BQError) as e:
        m.mlp_swiglu(x640, w(F, 640), w(F, 640), w(256, F))         # gate/up K not a multiple of 1024
    assert e.value.status_name == "BQ_ERR_SHAPE"
