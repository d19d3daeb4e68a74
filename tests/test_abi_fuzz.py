"""Random arguments into every entry point of the C ABI, on the CPU: each call must return one of
the documented status codes (or, for the size queries, a number) and never crash. Pointer
arguments are NULL, misaligned or aligned addresses that are never valid memory, so a call that
touched one on the host would fault; sizes, formats and dtypes range over valid and invalid
values. Without a GPU a call whose arguments pass validation stops at the first CUDA call
(BQ_ERR_CUDA or BQ_ERR_UNSUPPORTED); arguments that break a documented rule must be rejected
with its code before that. The calls run in a child process, so a crash fails this test instead
of the test run."""

import os
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(r"""
    import ctypes, sys
    import numpy as np
    sys.path.insert(0, ROOT)
    import ternary_g128_weight_bq_b200 as bq
    L = bq.lib()
    rng = np.random.default_rng(20260)
    PTRS = [0, 8, 24, 1 << 40, (1 << 40) + 16, (1 << 44) + 4096]
    def ptr(): return int(PTRS[rng.integers(len(PTRS))])
    def size(lo, hi): return int(rng.choice([lo - 1, lo, hi, hi + 1, int(rng.integers(lo, hi + 1)), 0, -1]))
    def kval(): return int(rng.choice([128, 1024, 5120, 20480, 1 << 24, (1 << 24) + 128, 100, 0, -128, 1 << 40]))
    def nval(): return int(rng.choice([1, 16, 5120, 248320, 1 << 31, (1 << 31) + 1, 0, -5, 1 << 50]))
    def weight():
        return bq._Weight(int(rng.integers(-1, 5)), nval(), kval(), ptr(), ptr())
    def valid_weight(w):
        words, scales = w.words or 0, w.scales or 0          # a NULL void* field reads as None
        return (w.fmt in (0, 1, 2) and 1 <= w.N <= (1 << 31) and 128 <= w.K <= (1 << 24) and w.K % 128 == 0
                and words != 0 and scales != 0 and words % 16 == 0 and scales % 16 == 0)
    def dt(): return int(rng.integers(-1, 7))
    ok_codes = set(range(0, 10))
    bad = []
    calls = 0
    for it in range(3000):
        w, w2, w3 = weight(), weight(), weight()
        W, W2, W3 = ctypes.byref(w), ctypes.byref(w2), ctypes.byref(w3)
        M = size(1, 8)
        r = {
            "gemv": L.bq_gemv(ptr(), dt(), M, W, ptr(), dt(), ptr(), int(rng.integers(0, 1 << 30)), None),
            "gemv_noalloc": L.bq_gemv_noalloc(ptr(), dt(), M, W, ptr(), dt(), None),
            "gemv_topk": L.bq_gemv_topk(ptr(), dt(), M, W, size(1, 32), ptr(), ptr(), ptr(), float(rng.uniform(-1, 2)),
                                        float(rng.uniform(-1, 2)), ptr(), ptr(), int(rng.integers(0, 1 << 30)), None),
            "mlp_swiglu": L.bq_mlp_swiglu(ptr(), dt(), M, W, W2, W3, ptr(), dt(), ptr(), int(rng.integers(0, 1 << 30)),
                                          None),
            "gemm_prefill": L.bq_gemm_prefill(ptr(), dt(), size(1, 4096), W, ptr(), dt(), ptr(),
                                              int(rng.integers(0, 1 << 30)), None),
            "embed_gather": L.bq_embed_gather(ptr(), size(0, 1 << 20), W, ptr(), dt(), None),
            "unpack": L.bq_unpack_g128(W, ptr(), ptr(), None),
            "pack_binary": L.bq_pack_binary_g128(ptr(), ptr(), nval(), kval(), ptr(), ptr(), None),
            "pack_ternary": L.bq_pack_ternary_g128(ptr(), ptr(), nval(), kval(), ptr(), ptr(), None),
            "pack_b3": L.bq_pack_ternary_b3_g128(ptr(), ptr(), nval(), kval(), ptr(), ptr(), None),
            "quantize": L.bq_quantize_g128(ptr(), dt(), nval(), kval(), int(rng.integers(-1, 5)), ptr(), ptr(), None),
        }
        for name, st in r.items():
            calls += 1
            if st not in ok_codes:
                bad.append((name, st))
        # documented rejections that come before any CUDA call
        if not valid_weight(w):
            for name in ("gemv", "gemv_noalloc", "gemv_topk", "gemm_prefill", "embed_gather", "unpack"):
                if r[name] in (0, 6, 8):
                    bad.append((name + " accepted an invalid weight view", w.fmt, w.N, w.K, w.words, w.scales))
        # the size queries return a number for any input
        for q in (L.bq_gemv_workspace_bytes(M, W), L.bq_gemv_topk_workspace_bytes(M, W, size(1, 32)),
                  L.bq_mlp_swiglu_workspace_bytes(M, W, W2, W3), L.bq_gemm_prefill_workspace_bytes(size(1, 4096), W),
                  L.bq_packed_words(int(rng.integers(-1, 5)), nval(), kval()),
                  L.bq_packed_bytes(int(rng.integers(-1, 5)), nval(), kval())):
            calls += 1
            if not isinstance(q, int) or q < 0:
                bad.append(("size query", q))
    print("calls", calls, "bad", len(bad))
    for b in bad[:20]:
        print(b)
    sys.exit(1 if bad else 0)
""").replace("ROOT", repr(ROOT))


def test_random_arguments_never_crash():
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "bad 0" in r.stdout
