"""Helpers shared by the GPU parity tests: input generation (from synth) and the
comparison against the CPU oracle. Nothing here computes an expected value itself."""

import numpy as np
import pytest
import torch

import oracle
import synth

requires_gpu = [pytest.mark.gpu,
                pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def bq():
    import ternary_g128_weight_bq_b200 as m
    from ternary_g128_weight_bq_b200 import build
    build.build()
    return m


def x_dtype_code(dt):
    return oracle.X_F16 if dt == torch.float16 else oracle.X_BF16


def binary_inputs(seed, N, K, M, xdt=torch.bfloat16):
    words = synth.binary_words(seed, N, K)                       # int32 bits [N, K/32]
    s = synth.scales(seed, N, K // 128)
    x = synth.activations(seed, M, K, dtype=xdt)
    return x, words, s


def ternary_q(seed, N, K):
    return synth.random_ternary(seed, synth.TID_TERNARY, (N, K))


def assert_within_bound(y_gpu, y_ref, bound, what=""):
    """max |y - y_ref| <= 2e-3 * sum_k |x s| per output (the bound the oracle computes)."""
    y = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    err = np.abs(y - y_ref)
    ratio = np.max(err / np.maximum(bound, 1e-300))
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    assert np.all(err <= bound), f"{what}: max err/bound = {ratio:.3g}"
    return float(ratio)


def sample_rows(N, count, seed=0):
    """Row indices to check at full size: the first and last rows plus a seeded sample."""
    rng = np.random.default_rng(seed)
    edge = np.array([0, 1, N // 2, N - 2, N - 1])
    pick = rng.choice(N, size=min(count, N), replace=False)
    return np.unique(np.clip(np.concatenate([edge, pick]), 0, N - 1)).astype(np.int64)
