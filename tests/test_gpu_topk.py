"""LM head fused with top-k (and the draw of a token) on the GPU.

* Against the CPU oracle: every returned value is within the GEMV bound of the oracle's logit
  of that index, the returned set is one the bound allows (every index whose oracle logit
  exceeds the k-th by more than the bounds is returned; every returned one could be in the top
  k), the order is descending; the drawn token is the oracle's draw on the returned candidates
  wherever u is not within 1e-4 of a boundary of the cumulative distribution.
* Against the plain GEMV kernel (same arithmetic, logits written out): indices and values
  identical to the k largest of its output, equal values by lower index.
Shapes: the 248 320-row LM head at K = 5120, a mid-size matrix, and rows per CTA fewer than k.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_common import bq, requires_gpu, ternary_q

pytestmark = requires_gpu


def weights(orc, fmt, seed, N, K):
    m = bq()
    s = synth.scales(seed, N, K // 128)
    if fmt == oracle.BINARY:
        words = synth.binary_words(seed, N, K)
        return m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda()), words.numpy(), s
    q = ternary_q(seed, N, K)
    if fmt == oracle.TERNARY:
        w = m.pack_ternary_g128(q.cuda(), s.cuda())
    else:
        w = m.pack_ternary_b3_g128(q.cuda(), s.cuda())
    st, ref, s_ref = orc.pack(fmt, q.numpy(), s.numpy())
    assert st == oracle.OK
    return w, ref, s_ref


def top_of(y, k):
    """k largest of each row of y (numpy), equal values by lower index."""
    out = []
    for row in y:
        order = np.lexsort((np.arange(len(row)), -row.astype(np.float64)))[:k]
        out.append(order)
    return np.array(out)


def check_against_oracle(orc, fmt, x, ref, s_ref, K, vals, idx, k):
    y_ref, bound = orc.gemv(fmt, x, oracle.X_BF16, ref, s_ref, K)
    M = y_ref.shape[0]
    for mrow in range(M):
        v, i = vals[mrow].astype(np.float64), idx[mrow]
        assert len(set(i.tolist())) == k, "indices repeat"
        assert np.all(np.diff(v) <= 0), "not descending"
        assert np.all(np.abs(v - y_ref[mrow, i]) <= bound[mrow, i]), "value outside the bound"
        oi, ov = orc.topk(y_ref[mrow:mrow + 1], k)
        kth = ov[0, -1]
        # every index certainly above the k-th must be returned
        sure = np.nonzero(y_ref[mrow] - bound[mrow] > kth + bound[mrow, oi[0, -1]])[0]
        assert set(sure.tolist()) <= set(i.tolist()), "a certain top-k index is missing"
        # every returned index could be in the top k
        assert np.all(y_ref[mrow, i] + bound[mrow, i] >= kth - bound[mrow, oi[0, -1]])


@pytest.mark.parametrize("k", [1, 20, 32])
def test_lm_head_topk_binary(orc, k):
    """The LM head (N = 248320, K = 5120), M = 1, binary: against the oracle and the plain GEMV."""
    m = bq()
    N, K = 248320, 5120
    w, ref, s_ref = weights(orc, oracle.BINARY, 0, N, K)
    x = synth.activations(0, 1, K)
    vals, idx = m.gemv_topk(x.cuda(), w, k=k)
    y = m.gemv(x.cuda(), w).cpu().numpy()
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    exp = top_of(y, k)
    assert np.array_equal(idx, exp) and np.array_equal(vals, np.take_along_axis(y, exp, axis=1))
    check_against_oracle(orc, oracle.BINARY, x, ref, s_ref, K, vals, idx, k)


@pytest.mark.parametrize("M", [5, 6, 8])
def test_lm_head_topk_batch(orc, M):
    """The LM head at M = 5, 6, 8: the CTAs' logits are too many for shared memory next to the
    pipeline, so the kernel keeps them in the workspace; same results as the plain GEMV."""
    m = bq()
    N, K, k = 248320, 5120, 20
    w = m.BQWeight(m.BINARY_G128, N, K, synth.binary_words(3, N, K).cuda(), synth.scales(3, N, K // 128).cuda())
    x = synth.activations(3 + M, M, K).cuda()
    vals, idx = m.gemv_topk(x, w, k=k)
    y = m.gemv(x, w).cpu().numpy()
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    exp = top_of(y, k)
    assert np.array_equal(idx, exp) and np.array_equal(vals, np.take_along_axis(y, exp, axis=1))


@pytest.mark.parametrize("fmt", [oracle.BINARY, oracle.TERNARY, oracle.TERNARY_B3])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_topk_matches_gemv(orc, fmt, M):
    """N = 20480, K = 5120: every M (one to four column sets), all three storages, k = 20."""
    m = bq()
    N, K, k = 20480, 5120, 20
    w, ref, s_ref = weights(orc, fmt, 40 + M, N, K)
    x = synth.activations(40 + M, M, K)
    vals, idx = m.gemv_topk(x.cuda(), w, k=k)
    y = m.gemv(x.cuda(), w).cpu().numpy()
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    exp = top_of(y, k)
    assert np.array_equal(idx, exp) and np.array_equal(vals, np.take_along_axis(y, exp, axis=1))


@pytest.mark.parametrize("N,k", [(40, 32), (17, 17), (1000, 32), (5000, 7)])
def test_topk_small_n_against_oracle(orc, N, k):
    """Few rows per CTA (fewer than k), every output checked against the oracle."""
    m = bq()
    K, M = 1024, 2
    w, ref, s_ref = weights(orc, oracle.TERNARY, 50 + N, N, K)
    x = synth.activations(50 + N, M, K)
    vals, idx = m.gemv_topk(x.cuda(), w, k=k)
    vals, idx = vals.cpu().numpy(), idx.cpu().numpy()
    check_against_oracle(orc, oracle.TERNARY, x, ref, s_ref, K, vals, idx, k)
    y = m.gemv(x.cuda(), w).cpu().numpy()
    assert np.array_equal(idx, top_of(y, k))


def test_topk_ties(orc):
    """Rows with identical weights give identical logits: the lower index comes first."""
    m = bq()
    N, K, k = 3000, 1024, 32
    words = synth.binary_words(60, N, K)
    words[1000:1100] = words[5]                      # 101 rows equal to row 5
    s = synth.scales(60, N, K // 128)
    s[1000:1100] = s[5]
    w = m.BQWeight(m.BINARY_G128, N, K, words.cuda(), s.cuda())
    x = synth.activations(60, 1, K)
    # make row 5 the largest: flip x to agree with its signs
    q, _ = orc.unpack(oracle.BINARY, words[5:6].numpy(), K)
    x = (torch.from_numpy(q.astype(np.float32)) * x.float().abs()).to(torch.bfloat16)
    vals, idx = m.gemv_topk(x.cuda(), w, k=k)
    idx = idx.cpu().numpy()[0]
    assert idx[0] == 5 and idx[1:].tolist() == list(range(1000, 1031))
    assert torch.all(vals[0] == vals[0, 0])


def test_topk_draw(orc):
    """Tokens drawn with the model card's settings (temperature 0.7, top-p 0.95) equal the
    oracle's draw from the same candidates, except where u lies within 1e-4 of a boundary."""
    m = bq()
    N, K, M, k = 20480, 5120, 8, 20
    w, ref, s_ref = weights(orc, oracle.BINARY, 70, N, K)
    for trial in range(6):
        x = synth.activations(70 + trial, M, K)
        u = torch.rand(M, generator=torch.Generator().manual_seed(trial), dtype=torch.float32)
        vals, idx, tok = m.gemv_topk(x.cuda(), w, k=k, u=u.cuda(), temperature=0.7, top_p=0.95)
        vals, idx, tok = vals.cpu().numpy(), idx.cpu().numpy(), tok.cpu().numpy()
        for r in range(M):
            v = vals[r].astype(np.float64)
            lo = orc.sample_topk(v, idx[r], 0.7, 0.95, max(float(u[r]) - 1e-4, 0.0))
            hi = orc.sample_topk(v, idx[r], 0.7, 0.95, min(float(u[r]) + 1e-4, 0.999999))
            got = int(tok[r])
            if lo == hi:
                assert got == lo
            else:
                assert got in (lo, hi)


def test_topk_draw_extremes(orc):
    """top_p tiny keeps only the best candidate; u near 0 draws the first kept, near 1 the last."""
    m = bq()
    N, K = 4096, 1024
    w, _, _ = weights(orc, oracle.BINARY, 80, N, K)
    x = synth.activations(80, 2, K).cuda()
    u = torch.tensor([0.999, 0.0], device="cuda")
    vals, idx, tok = m.gemv_topk(x, w, k=20, u=u, temperature=0.7, top_p=1e-6)
    assert torch.equal(tok, idx[:, 0])
    vals, idx, tok = m.gemv_topk(x, w, k=20, u=torch.zeros(2, device="cuda"), temperature=0.7, top_p=1.0)
    assert torch.equal(tok, idx[:, 0])


def test_topk_deterministic():
    m = bq()
    N, K = 20480, 5120
    w = m.BQWeight(m.BINARY_G128, N, K, synth.binary_words(90, N, K).cuda(), synth.scales(90, N, K // 128).cuda())
    x = synth.activations(90, 4, K).cuda()
    v1, i1 = m.gemv_topk(x, w, k=32)
    for _ in range(5):
        v2, i2 = m.gemv_topk(x, w, k=32)
        assert torch.equal(v1, v2) and torch.equal(i1, i2)


def test_topk_errors():
    m = bq()
    w = m.BQWeight(m.BINARY_G128, 256, 1024, synth.binary_words(1, 256, 1024).cuda(), synth.scales(1, 256, 8).cuda())
    x = synth.activations(1, 1, 1024).cuda()
    vals = torch.empty((1, 40), device="cuda")
    idx = torch.empty((1, 40), dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    for k in (0, 33):
        with pytest.raises(m.BQError) as e:
            m._check(m.lib().bq_gemv_topk(x.data_ptr(), 1, 1, w.c, k, vals.data_ptr(), idx.data_ptr(), None, 0.7,
                                          0.95, None, ws.data_ptr(), ws.numel(), m._stream()))
        assert e.value.status_name == "BQ_ERR_SHAPE"
    w640 = m.BQWeight(m.BINARY_G128, 256, 640, synth.binary_words(1, 256, 640).cuda(), synth.scales(1, 256, 5).cuda())
    with pytest.raises(m.BQError) as e:
        m.gemv_topk(synth.activations(1, 1, 640).cuda(), w640, k=20)
    assert e.value.status_name == "BQ_ERR_SHAPE"
    assert m.gemv_topk_workspace_bytes(1, w640, 20) == 0
    with pytest.raises(m.BQError) as e:
        m.gemv_topk(x, w, k=20, u=torch.rand(1, device="cuda"), temperature=0.0)
    assert e.value.status_name == "BQ_ERR_INVALID_ARG"
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    vals = torch.empty((1, 20), device="cuda")
    idx = torch.empty((1, 20), dtype=torch.int32, device="cuda")
    with pytest.raises(m.BQError) as e:
        m._check(m.lib().bq_gemv_topk(x.data_ptr(), 1, 1, w.c, 20, vals.data_ptr(), idx.data_ptr(), None, 0.7, 0.95,
                                      None, small.data_ptr(), 16, m._stream()))
    assert e.value.status_name == "BQ_ERR_WORKSPACE"
